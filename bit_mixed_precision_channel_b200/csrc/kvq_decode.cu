// kvq_decode.cu — decode attention over the paged 2-bit cache, sm_100a.
//
// One CTA = (sequence b, kv head, split of the page list); 4 warps.  Pages stream
// through a 6-stage shared-memory ring filled by the bulk-copy engine (one
// cp.async.bulk per page record, completion on an mbarrier, L2 evict-first hint);
// a stage holds 128 tokens (1, 2 or 4 pages).  Each warp owns one 32-token key
// group of the stage and keeps its own online-softmax state; the warps' states are
// merged in shared memory at the end, and the splits of a sequence are merged by the
// last CTA to finish (log-sum-exp merge, no second launch).
//
// The 2-bit codes never become floating-point values with a scale applied.  The
// scales are folded into the other operand of each product, and the codes go to the
// tensor cores as they are (Kitty abstract: page dequantization kernels with uniform
// 2-bit dequantization; MiniKV proposed method: dequantization fused into the matmul):
//   q.k_t   = sum_c code_A[t,c] * (q_c * sA_{g,c}) + sum_j code_B[t,j] * (q_{idx_j} * sB_{g,j})
//             + sum_c q_c * zA_{g,c}
//   sum_t p_t v_t[c] = sum_t code_V[t,c] * (p_t * sV_t) + sum_t p_t * zV_t
// With the 4-bit boosted channels stored as two 2-bit planes, the boosted low bits
// are simply 16*(k/16) more rows of the same contraction.  The folded operands are
// carried as a high and a low fp16 part (hi = fp16(x), lo = fp16(x - hi)), so the
// products keep ~22 bits; codes are exact in fp16.  Matrix shapes per warp and
// 32-token group: QK^T = [32 tokens x (128 + k) channels] x [(128 + k) x 8 columns],
// PV = [128 channels x 32 tokens] x [32 tokens x 8 columns], where the 8 columns hold
// the hi and lo parts of up to 4 query heads (two column tiles for 8 heads).
#include <algorithm>

#include "kvq_internal.cuh"

namespace kvq {

constexpr int kStages = 6;
constexpr int kDecodeThreads = 128;
constexpr int kResRowBytes = 272;  // residual row in shared memory: 256 bytes + 16 pad

// ---------------------------------------------------------------- operand builders

// Query-side operand of one k-step pair for the quantized planes:
// hi = fp16(q*s) and lo = fp16(q*s - hi).  For fp16 data the product of two fp16
// values is exact in 22 bits; hmul2 rounds it once and hfma2 returns the rest.
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

// Online-softmax update from the 2 x 4 logits of one 32-token group held by this
// lane (rows g, g+8 of two 16-token tiles; heads hc0, hc1).  Logits are in log2 units.
template <int GQA>
__device__ __forceinline__ void softmax_step(WarpState<GQA>& st, const float (&L)[2][4], float (&alpha)[2]) {
  float mx[2];
  mx[0] = fmaxf(fmaxf(L[0][0], L[0][2]), fmaxf(L[1][0], L[1][2]));
  mx[1] = fmaxf(fmaxf(L[0][1], L[0][3]), fmaxf(L[1][1], L[1][3]));
#pragma unroll
  for (int j = 0; j < 2; ++j) {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) mx[j] = fmaxf(mx[j], __shfl_xor_sync(kFull, mx[j], off));
    const float mn = fmaxf(st.m[j], mx[j]);
    alpha[j] = (mn == -INFINITY) ? 1.0f : ex2(st.m[j] - mn);
    st.m[j] = mn;
    st.l[j] *= alpha[j];
    st.zv[j] *= alpha[j];
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
template <typename T, int GQA>
__device__ __forceinline__ void page_group(const DecodeParams& p, const uint8_t* rec, int t0,
                                           const uint32_t (&qv)[8][2], const T* q_s, int hB, bool loB,
                                           bool validB, WarpState<GQA>& st, int g, int qd) {
  constexpr int NT = WarpState<GQA>::NT;
  const int grp = t0 >> 5;
  float acc[2][NT][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.0f;

  // -- q . K^T over plane A (128 channels) --
  const uint8_t* kA = rec + p.L.k_codes;
  const uint8_t* ksc = rec + p.L.k_scale + grp * kHeadDim * 2;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint4 w[2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int r = 0; r < 2; ++r) w[mt][r] = lds128(kA + ((t0 + 16 * mt + g + 8 * r) * 8 + 4 * half) * 4);
#pragma unroll
    for (int ss = 0; ss < 4; ++ss) {
      const int s = 4 * half + ss;
      const uint32_t sc0 = lds32(ksc + (16 * s + 2 * qd) * 2);
      const uint32_t sc1 = lds32(ksc + (16 * s + 2 * qd + 8) * 2);
      uint32_t h0, l0, h1, l1;
      fold_hilo(qv[s][0], sc0, h0, l0, T());
      fold_hilo(qv[s][1], sc1, h1, l1, T());
      uint32_t b[NT][2];
      if constexpr (NT == 1) {
        b[0][0] = loB ? l0 : h0;
        b[0][1] = loB ? l1 : h1;
      } else {
        b[0][0] = h0; b[0][1] = h1;
        b[1][0] = l0; b[1][1] = l1;
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const uint32_t wa = ss == 0 ? w[mt][0].x : ss == 1 ? w[mt][0].y : ss == 2 ? w[mt][0].z : w[mt][0].w;
        const uint32_t wb = ss == 0 ? w[mt][1].x : ss == 1 ? w[mt][1].y : ss == 2 ? w[mt][1].z : w[mt][1].w;
        const uint32_t a[4] = {code_pair(wa, qd), code_pair(wb, qd), code_pair(wa, qd + 4), code_pair(wb, qd + 4)};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_16816(acc[mt][nt], a, b[nt][0], b[nt][1], __half());
      }
    }
  }
  // -- plane B: low bits of the boosted channels (k rows) --
  const uint8_t* kB = rec + p.L.kb_codes;
  const uint8_t* idx = rec + p.L.boost_idx;
  const uint8_t* kbsc = rec + p.L.kb_scale + grp * p.k * 2;
  for (int s = 0; s < p.KB; ++s) {
    const int j0 = 16 * s + 2 * qd, j1 = j0 + 8;
    const uint16_t* qh = reinterpret_cast<const uint16_t*>(q_s) + hB * kHeadDim;
    uint32_t q0 = 0, q1 = 0;
    if (validB) {
      // indices are < 128 in any record the library wrote; the mask keeps a corrupt
      // record from reading outside the query rows
      q0 = uint32_t(qh[idx[j0] & 127]) | (uint32_t(qh[idx[j0 + 1] & 127]) << 16);
      q1 = uint32_t(qh[idx[j1] & 127]) | (uint32_t(qh[idx[j1 + 1] & 127]) << 16);
    }
    uint32_t h0, l0, h1, l1;
    fold_hilo(q0, lds32(kbsc + j0 * 2), h0, l0, T());
    fold_hilo(q1, lds32(kbsc + j1 * 2), h1, l1, T());
    uint32_t b[NT][2];
    if constexpr (NT == 1) {
      b[0][0] = loB ? l0 : h0;
      b[0][1] = loB ? l1 : h1;
    } else {
      b[0][0] = h0; b[0][1] = h1;
      b[1][0] = l0; b[1][1] = l1;
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      const uint32_t wa = lds32(kB + ((t0 + 16 * mt + g) * p.KB + s) * 4);
      const uint32_t wb = lds32(kB + ((t0 + 16 * mt + g + 8) * p.KB + s) * 4);
      const uint32_t a[4] = {code_pair(wa, qd), code_pair(wb, qd), code_pair(wa, qd + 4), code_pair(wb, qd + 4)};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_16816(acc[mt][nt], a, b[nt][0], b[nt][1], __half());
    }
  }
  // -- zero-point term: Z[h] = sum_c q[h][c] * zA[g][c] (rows of A all equal) --
  float z[4] = {0.f, 0.f, 0.f, 0.f};
  {
    const uint8_t* kzp = rec + p.L.k_zero + grp * kHeadDim * 2;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint32_t z0 = lds32(kzp + (16 * s + 2 * qd) * 2);
      const uint32_t z1 = lds32(kzp + (16 * s + 2 * qd + 8) * 2);
      const uint32_t a[4] = {z0, z0, z1, z1};
      const bool useq = validB && !loB;
      mma_16816(z, a, useq ? qv[s][0] : 0u, useq ? qv[s][1] : 0u, T());
    }
  }
  // -- logits (log2 units) --
  float L[2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v;
      if constexpr (NT == 1) {
        v = (acc[mt][0][i] + z[i & 1]) * p.c_log2;
        v += __shfl_xor_sync(kFull, v, 2);
      } else {
        v = (acc[mt][0][i] + acc[mt][1][i] + z[i & 1]) * p.c_log2;
      }
      L[mt][i] = v;
    }
  float alpha[2];
  softmax_step<GQA>(st, L, alpha);

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
  // -- P V over the value codes (channel-major words of 16 tokens) --
  const uint8_t* vq = rec + p.L.v_codes;
  const int PW = p.P >> 4;
#pragma unroll
  for (int mc = 0; mc < 8; ++mc) {
    const uint2 w0 = lds64(vq + ((16 * mc + g) * PW + (t0 >> 4)) * 4);
    const uint2 w1 = lds64(vq + ((16 * mc + g + 8) * PW + (t0 >> 4)) * 4);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const uint32_t wa = ks ? w0.y : w0.x, wb = ks ? w1.y : w1.x;
      const uint32_t a[4] = {code_pair(wa, qd), code_pair(wb, qd), code_pair(wa, qd + 4), code_pair(wb, qd + 4)};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_16816(st.o[mc][nt], a, pb[ks][nt][0], pb[ks][nt][1], __half());
    }
  }
}

// ---------------------------------------------------------------- residual group

// Tokens [tw, tw+32) of the residual window staged in shared memory (rows of 272 B);
// rows at or beyond rl are zero and masked out of the softmax.
template <typename T, int GQA>
__device__ __forceinline__ void residual_group(const DecodeParams& p, const uint8_t* Kr, const uint8_t* Vr,
                                               int tw, int rl, const uint32_t (&qv)[8][2], bool loB,
                                               bool validB, WarpState<GQA>& st, int lane, int g, int qd) {
  constexpr int NT = WarpState<GQA>::NT;
  float acc[2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[mt][i] = 0.0f;
  const bool useq = validB && !loB;
  const int li = lane >> 3, lr = lane & 7;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      uint32_t a[4];
      const int row = tw + 16 * mt + lr + 8 * (li & 1);
      const int col = 16 * s + 8 * (li >> 1);
      ldmatrix_x4(a, smem_addr(Kr + row * kResRowBytes + col * 2));
      mma_16816(acc[mt], a, useq ? qv[s][0] : 0u, useq ? qv[s][1] : 0u, T());
    }
  }
  float L[2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v = acc[mt][i] * p.c_log2;
      if constexpr (NT == 1) v += __shfl_xor_sync(kFull, v, 2);
      const int tok = tw + 16 * mt + g + 8 * (i >> 1);
      L[mt][i] = tok < rl ? v : -INFINITY;
    }
  float alpha[2];
  softmax_step<GQA>(st, L, alpha);
  uint32_t pb[2][NT][2];
  const bool loC = qd >= 2;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    const float p00 = ex2(L[mt][0] - st.m[0]), p01 = ex2(L[mt][1] - st.m[1]);
    const float p10 = ex2(L[mt][2] - st.m[0]), p11 = ex2(L[mt][3] - st.m[1]);
    st.l[0] += p00 + p10;
    st.l[1] += p01 + p11;
    uint32_t th, tl, bh, bl;
    split_t(p00, p01, th, tl, T());
    split_t(p10, p11, bh, bl, T());
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
#pragma unroll
  for (int mc = 0; mc < 8; ++mc)
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t a[4];
      const int row = tw + 16 * ks + lr + 8 * (li >> 1);
      const int col = 16 * mc + 8 * (li & 1);
      ldmatrix_x4_trans(a, smem_addr(Vr + row * kResRowBytes + col * 2));
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_16816(st.o[mc][nt], a, pb[ks][nt][0], pb[ks][nt][1], T());
    }
}

// ---------------------------------------------------------------- the kernel

template <typename T, int GQA>
__global__ void __launch_bounds__(kDecodeThreads, 2) decode_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int NT = WarpState<GQA>::NT;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t bars[kStages];
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
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    s_abort = 0;
  }
  __syncthreads();

  const int ppc = 128 / p.P;
  const int n_chunks = (npg + ppc - 1) / ppc;
  const uint64_t policy = l2_evict_first_policy();
  auto issue = [&](int c) {
    const int st = c % kStages, first = c * ppc, nv = min(ppc, npg - first);
    mbar_arrive_expect_tx(&bars[st], uint32_t(nv) * p.payload);
    for (int i = 0; i < nv; ++i) {
      const uint8_t* src = p.pool + (size_t(s_pages[first + i]) * p.Hkv + kvh) * p.rec_bytes;
      bulk_g2s(main + st * p.stage_bytes + i * p.rec_bytes, src, p.payload, &bars[st], policy);
    }
  };
  int issued = 0;
  if (tid == 0) {
    for (; issued < min(kStages - 1, n_chunks); ++issued) issue(issued);
  }

  // query fragments of this lane's B column (head hB; lo part for columns 4..7 when GQA <= 4)
  const int hB = GQA <= 4 ? (g & 3) : g;
  const bool loB = GQA <= 4 && g >= 4;
  const bool validB = hB < GQA;
  uint32_t qv[8][2];
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    qv[s][0] = validB ? lds32(q_s + hB * kHeadDim + 16 * s + 2 * qd) : 0u;
    qv[s][1] = validB ? lds32(q_s + hB * kHeadDim + 16 * s + 2 * qd + 8) : 0u;
  }

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
  int consumed = 0;
  for (int c = 0; c < n_chunks; ++c) {
    __syncthreads();  // every warp is done with chunk c-1; its stage may be refilled
    if (s_abort) break;
    if (tid == 0 && issued < n_chunks) issue(issued++);
    const int stg = c % kStages;
    if (!mbar_wait_bounded(&bars[stg], uint32_t(c / kStages) & 1u)) {
      flag_error(p.err, KVQ_DEV_ERR_TIMEOUT);
      s_abort = 1;
      continue;
    }
    consumed = c + 1;
    if (c * ppc + pi < npg)
      page_group<T, GQA>(p, main + stg * p.stage_bytes + pi * p.rec_bytes, t0, qv,
                         reinterpret_cast<const T*>(q_s), hB, loB, validB, st, g, qd);
  }
  __syncthreads();
  if (s_abort) {
    // drain the copies still in flight (bounded), then leave; the output is undefined
    if (tid == 0)
      for (int c = consumed; c < issued; ++c) mbar_wait_bounded(&bars[c % kStages], uint32_t(c / kStages) & 1u);
    __syncthreads();
    return;
  }
  // ---------------------------------------------------------------- residual window
  if (own_res) {
    const int rows = (rl + 31) & ~31;
    uint8_t* Kr = main;
    uint8_t* Vr = main + p.P * kResRowBytes;
    const uint8_t* gk = reinterpret_cast<const uint8_t*>(p.res_k + (size_t(b) * p.Hkv + kvh) * p.P * kHeadDim);
    const uint8_t* gv = reinterpret_cast<const uint8_t*>(p.res_v + (size_t(b) * p.Hkv + kvh) * p.P * kHeadDim);
    for (int i = tid; i < rows * 32; i += kDecodeThreads) {
      const int which = i / (rows * 16), j = i % (rows * 16), t = j >> 4, c16 = j & 15;
      const uint8_t* src = (which ? gv : gk) + t * 256 + c16 * 16;
      uint8_t* dst = (which ? Vr : Kr) + t * kResRowBytes + c16 * 16;
      cp_async16(dst, t < rl ? src : gk, t < rl ? 16u : 0u);
    }
    cp_async_wait_all();
    __syncthreads();
    const int tw = 32 * warp;
    if (tw < rl) residual_group<T, GQA>(p, Kr, Vr, tw, rl, qv, loB, validB, st, lane, g, qd);
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

// Pages per split: minimises waves x (pages per CTA + startup), where a wave is
// 2 resident CTAs per SM and the startup cost of a CTA is about 4 pages of streaming.
SplitPlan plan_splits(int units, int max_pages, int sm_count) {
  SplitPlan best{max(max_pages, 1), 1};
  if (max_pages <= 1 || units <= 0) return best;
  const long long slots = 2ll * sm_count;
  double best_cost = 1e300;
  const int min_splits = (max_pages + 2047) / 2048;  // page-id list fits in 8 KB of shared memory
  for (int s = max(1, min_splits); s <= min(max_pages, 64); ++s) {
    const int pps = (max_pages + s - 1) / s;
    const int se = (max_pages + pps - 1) / pps;
    const long long ctas = 1ll * units * se;
    const long long waves = (ctas + slots - 1) / slots;
    const double cost = double(waves) * (pps + 4);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = {pps, se};
    }
  }
  return best;
}

size_t decode_main_bytes(int P, int GQA, uint32_t rec_bytes) {
  const size_t stage = size_t(128 / P) * rec_bytes;
  size_t m = kStages * stage;
  m = std::max(m, size_t(P) * 2 * kResRowBytes);
  m = std::max(m, size_t(4) * GQA * kHeadDim * 4);
  return (m + 127) / 128 * 128;
}

template <typename T, int GQA>
cudaError_t launch_decode_t(DecodeParams p, cudaStream_t stream) {
  const size_t smem = size_t(p.main_bytes) + size_t(p.pps) * 4;
  static int seen[64];
  cudaError_t e = ensure_dynamic_smem(decode_kernel<T, GQA>, int(smem), seen);
  if (e != cudaSuccess) return e;
  const dim3 grid(p.max_splits, p.Hkv, p.batch);
  decode_kernel<T, GQA><<<grid, kDecodeThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeParams& p, int gqa, int dtype, cudaStream_t stream) {
  if (p.batch <= 0) return cudaSuccess;
  if (dtype == KVQ_BF16) {
    switch (gqa) {
      case 1: return launch_decode_t<__nv_bfloat16, 1>(p, stream);
      case 2: return launch_decode_t<__nv_bfloat16, 2>(p, stream);
      case 4: return launch_decode_t<__nv_bfloat16, 4>(p, stream);
      case 8: return launch_decode_t<__nv_bfloat16, 8>(p, stream);
    }
  } else {
    switch (gqa) {
      case 1: return launch_decode_t<__half, 1>(p, stream);
      case 2: return launch_decode_t<__half, 2>(p, stream);
      case 4: return launch_decode_t<__half, 4>(p, stream);
      case 8: return launch_decode_t<__half, 8>(p, stream);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace kvq
