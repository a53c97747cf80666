// kvq_quantize.cu — page quantization (boost selection, two-plane keys, per-token
// values), residual append and residual flush for sm_100a.
//
// One CTA quantizes one (page, kv head): it stages the page's K and V tiles
// ([P][128] each) in shared memory with 16-byte loads, then
//   a1  ranks channels by max |K| over the page (Kitty, Dynamic Channel-wise
//       Precision Boost; magnitude heuristic per the notes.yuuk.io wiki page),
//   a2  quantizes every (key group, channel) asymmetrically — 4 bits for boosted
//       channels, split into a high plane and a low plane of 2-bit codes, 2 bits
//       otherwise (KIVI per-channel keys; Kitty two uniform 2-bit tensors),
//   a3  quantizes every token's values over the head dimension (KIVI per-token values),
// and writes the packed record.  The quantizer's fp32 operations use explicit
// round-to-nearest intrinsics in the order the ABI documents, so codes, scales and
// zeros are bit-identical to any implementation of that definition.
#include "kvq_internal.cuh"

namespace kvq {

constexpr int kQThreads = 256;

// Shared memory of one quantize CTA.  A CTA quantizes either the keys of a (page, kv
// head) (selection and both planes) or its values, so that four CTAs fit on an SM.
struct QSmem {
  static size_t key_bytes(int P, int k) {
    return size_t(P) * kHeadDim * 2        // K tile
           + size_t(P) * kHeadDim          // plane-A codes [P][128]
           + size_t(P) * (k > 0 ? k : 16)  // plane-B codes [P][k]
           + 16                            // scratch byte of channels that are not boosted
           + kHeadDim * 4 * 2 + 16 * 4;    // scores, plane-B row of each channel, warp counts
  }
  static size_t value_bytes(int P) {
    return size_t(P) * kHeadDim * 2  // V tile
           + size_t(P) * kHeadDim;   // value codes [P][128]
  }
  static size_t bytes(int P, int k, int mode) {
    size_t b = 0;
    if (mode & (kModeSelect | kModeKeys)) b = key_bytes(P, k);
    if (mode & kModeValues) b = b > value_bytes(P) ? b : value_bytes(P);
    return b;
  }
};

// 16 codes given by element order (one byte each) -> one word, element e = 8a + 2b + f
// at bit 8b + 4f + 2a.  Bytes 4i..4i+3 (element 4i + m) land at bit
// 16*(i & 1) + 2*(i >> 1) + 4*m.
__device__ __forceinline__ uint32_t pack16(const uint8_t* c) {
  const uint4 v = lds128(c);
  const uint32_t q[4] = {v.x, v.y, v.z, v.w};
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t x = q[i];
    const uint32_t nib = (x & 0x3u) | ((x >> 4) & 0x30u) | ((x >> 8) & 0x300u) | ((x >> 12) & 0x3000u);
    w |= nib << (16 * (i & 1) + 2 * (i >> 1));
  }
  return w;
}

// Quantizes one group with the documented fp32 op order; returns the scale as float
// and writes scale/zero bits.  min/max are exact; a zero minimum is stored as +0.
template <typename T>
__device__ __forceinline__ float quant_params(float mn, float mx, int qmax, uint16_t& sbits, uint16_t& zbits,
                                              float& zero) {
  // +0 for a group of zeros whatever the signs the min/max kept (x - x is +0 too)
  const float range = __fsub_rn(__fadd_rn(mx, 0.0f), __fadd_rn(mn, 0.0f));
  const float s32 = __fdiv_rn(range, float(qmax));
  sbits = round_up_bits(s32, T());
  zero = __fadd_rn(mn, 0.0f);  // -0 -> +0
  zbits = exact_bits(zero, T());
  return bits_to_float(sbits, T());
}

__device__ __forceinline__ int quant_code(float x, float zero, float scale, int qmax) {
  if (scale == 0.0f) return 0;
  const float t = __fdiv_rn(__fsub_rn(x, zero), scale);
  float r = rintf(t);
  r = fminf(fmaxf(r, 0.0f), float(qmax));
  return int(r);
}

// Reciprocal of a group's scale for quant_bits_fma, or 0 when the fast path may not be
// used (scale 0, or below the smallest normal float, where the approximate reciprocal
// flushes).
__device__ __forceinline__ float quant_rcp(float scale) {
  if (!(scale >= 1.17549435e-38f)) return 0.0f;
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(scale));
  return r;
}

// The code quant_code gives, bit for bit, without a divide in almost every case.
// x - zero >= 0, and scale >= (max - min) / qmax (rounded up), so x - zero <= qmax * scale
// and no code exceeds qmax: the clamp never acts.  fma(d, rcp, 1.5 * 2^23) rounds the
// exact product d * rcp to an integer n held in the low byte of the result's bits
// (0x4B400000 + n, returned).  d * rcp is within 2^-17 of the correctly rounded quotient
// (rcp.approx: relative error below 2^-22; the divide: half an ulp, at most 2^-20), so n
// is the code unless d * rcp lies within 2^-14 of a rounding boundary n +- 1/2.  There
// `near` is set and the caller redoes the element with quant_code.  With rcp = 0
// (scale 0) the code is 0, as quant_code gives.
__device__ __forceinline__ uint32_t quant_bits_fma(float x, float zero, float rcp, bool& near) {
  const float d = __fsub_rn(x, zero);
  const float t = __fmaf_rn(d, rcp, 12582912.0f);
  const float res = __fmaf_rn(d, rcp, -__fsub_rn(t, 12582912.0f));
  near = !(fabsf(res) < 0.5f - 1.0f / 16384.0f);
  return __float_as_uint(t);
}

template <typename T>
__global__ void __launch_bounds__(kQThreads) quantize_kernel(const QuantParams p) {
  pdl_wait();
  const int item = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int P = p.P, k = p.k;
  int dst;
  if (p.flush) {
    if (p.res_len[item] != P) return;
    dst = p.dst_pages[item];
    const int np = p.num_pages[item];
    if (dst < 0 || np < 0 || np >= p.max_pages) {
      if (tid == 0 && h == 0) flag_error(p.err, KVQ_DEV_ERR_TABLE_FULL);
      return;
    }
  } else {
    dst = p.dst_pages[item];
  }
  if (dst < 0 || dst >= p.pool_pages) {
    if (tid == 0) flag_error(p.err, KVQ_DEV_ERR_PAGE_RANGE);
    return;
  }
  uint8_t* rec = p.pool + (size_t(dst) * p.Hkv + h) * p.L.record;

  // z = 0: the key part of the requested modes, z = gridDim.z - 1: the value part
  const int kmodes = blockIdx.z == 0 ? p.mode & (kModeSelect | kModeKeys) : 0;
  const int mode = kmodes | (blockIdx.z == gridDim.z - 1 ? p.mode & kModeValues : 0);
  const bool need_k = kmodes != 0;
  const bool need_v = mode & kModeValues;

  extern __shared__ __align__(16) uint8_t smem[];
  // key part: K tile, plane A codes [token][key position], plane B codes [token][boost
  // position], scores; value part: V tile, value codes [token][channel]
  uint16_t* Ks = reinterpret_cast<uint16_t*>(smem);
  uint8_t* cA = reinterpret_cast<uint8_t*>(Ks + P * kHeadDim);
  uint8_t* cB = cA + P * kHeadDim;
  uint8_t* cScratch = cB + P * (k > 0 ? k : 16);  // plane-B bytes of channels that are not boosted
  float* score = reinterpret_cast<float*>(cScratch + 16);
  int* row_of = reinterpret_cast<int*>(score + kHeadDim);
  int* warp_cnt = row_of + kHeadDim;
  uint16_t* Vs = reinterpret_cast<uint16_t*>(smem);
  uint8_t* cV = reinterpret_cast<uint8_t*>(Vs + P * kHeadDim);
  // boosted channels of this kv head: k, or the per-head count (plane-B rows kb..k-1,
  // their scales and indices then stay zero)
  int kb = k;
  if (p.kh && need_k) {
    kb = p.kh[h];
    if (kb < 0 || kb > k) {
      if (tid == 0) flag_error(p.err, KVQ_DEV_ERR_LENGTH);
      kb = kb < 0 ? 0 : k;
    }
  }

  // ---- stage the page tiles (rows of 128 x 16-bit = 16 x 16 bytes)
  if (need_k) {
    const uint16_t* src = p.k_src + item * p.k_page_stride + h * p.k_head_stride;
    for (int i = tid; i < P * 16; i += kQThreads) {
      const int t = i >> 4, c = i & 15;
      reinterpret_cast<uint4*>(Ks)[i] = __ldg(reinterpret_cast<const uint4*>(src + t * p.k_tok_stride) + c);
    }
  }
  if (need_v) {
    const uint16_t* src = p.v_src + item * p.v_page_stride + h * p.v_head_stride;
    for (int i = tid; i < P * 16; i += kQThreads) {
      const int t = i >> 4, c = i & 15;
      reinterpret_cast<uint4*>(Vs)[i] = __ldg(reinterpret_cast<const uint4*>(src + t * p.v_tok_stride) + c);
    }
  }
  __syncthreads();

  // ---- a1: boosted channels (or read them back from the record)
  if (mode & kModeSelect) {
    using T2 = typename Pair<T>::type;
    // score_c = max |K[t][c]| (magnitude), or fp32(w_c * fp32(max - min)) (query-aware):
    // thread = (channel pair tid / 4, token quarter tid % 4), packed abs/min/max (exact),
    // then the four quarters by shuffles
    {
      const int pr = tid >> 2, qt = tid & 3;
      const uint32_t* col = reinterpret_cast<const uint32_t*>(Ks) + pr;
      const int tq = P / 4;
      if (!p.qw) {
        T2 m = __habs2(u32_as_pair(col[qt * tq * (kHeadDim / 2)], T()));
#pragma unroll 8
        for (int t = 1; t < tq; ++t) m = __hmax2(m, __habs2(u32_as_pair(col[(qt * tq + t) * (kHeadDim / 2)], T())));
        uint32_t mb = pair_as_u32(m);
#pragma unroll
        for (int off = 1; off < 4; off <<= 1)
          mb = pair_as_u32(__hmax2(u32_as_pair(mb, T()), u32_as_pair(__shfl_xor_sync(kFull, mb, off), T())));
        if (qt == 0) {
          score[2 * pr] = bits_to_float(uint16_t(mb), T());
          score[2 * pr + 1] = bits_to_float(uint16_t(mb >> 16), T());
        }
      } else {
        T2 lo = u32_as_pair(col[qt * tq * (kHeadDim / 2)], T()), hi = lo;
#pragma unroll 8
        for (int t = 1; t < tq; ++t) {
          const T2 v = u32_as_pair(col[(qt * tq + t) * (kHeadDim / 2)], T());
          lo = __hmin2(lo, v);
          hi = __hmax2(hi, v);
        }
        uint32_t lb = pair_as_u32(lo), hb = pair_as_u32(hi);
#pragma unroll
        for (int off = 1; off < 4; off <<= 1) {
          lb = pair_as_u32(__hmin2(u32_as_pair(lb, T()), u32_as_pair(__shfl_xor_sync(kFull, lb, off), T())));
          hb = pair_as_u32(__hmax2(u32_as_pair(hb, T()), u32_as_pair(__shfl_xor_sync(kFull, hb, off), T())));
        }
        if (qt == 0) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float range = __fsub_rn(bits_to_float(uint16_t(hb >> (16 * e)), T()),
                                          bits_to_float(uint16_t(lb >> (16 * e)), T()));
            score[2 * pr + e] = __fmul_rn(p.qw[h * kHeadDim + 2 * pr + e], range);
          }
        }
      }
    }
    __syncthreads();
    // rank of channel c: channels with a higher score, or an equal score and a lower
    // index; two threads per channel (channels c' < 64 and >= 64), summed by a shuffle
    {
      const int c = tid >> 1, half = tid & 1;
      const float sc = score[c];
      int rank = 0;
#pragma unroll 8
      for (int i = 0; i < kHeadDim / 2; ++i) {
        const int o = half * (kHeadDim / 2) + i;
        const float so = score[o];
        rank += (so > sc) || (so == sc && o < c);
      }
      rank += __shfl_xor_sync(kFull, rank, 1);
      const bool boosted = rank < kb;
      // plane-B row of a boosted channel: boosted channels with a lower index before it
      const unsigned ballot = __ballot_sync(kFull, boosted && half == 0);
      if ((tid & 31) == 0) warp_cnt[tid >> 5] = __popc(ballot);
      __syncthreads();
      if (half == 0) {
        int before = 0;
        for (int w = 0; w < (tid >> 5); ++w) before += warp_cnt[w];
        const int row = boosted ? before + int(__popc(ballot & ((1u << (tid & 31)) - 1u))) : -1;
        row_of[c] = row;
        if (row >= 0) rec[p.L.boost_idx + row] = uint8_t(c);
      }
      if (tid >= kb && tid < k) rec[p.L.boost_idx + tid] = 0;  // unused rows
    }
    __syncthreads();
  } else if (mode & kModeKeys) {
    if (tid < kHeadDim) row_of[tid] = -1;
    __syncthreads();
    if (tid < kb) {
      const int c = rec[p.L.boost_idx + tid];
      if (c < kHeadDim) row_of[c] = tid;
    }
    __syncthreads();
  }

  // ---- a2: keys, one task per (group, pair of adjacent channels): 32-bit loads and
  //      packed min/max (exact) over the group's tokens
  if (mode & kModeKeys) {
    using T2 = typename Pair<T>::type;
    const int n_groups = P / kKeyGroup;
    uint16_t* ks_out = reinterpret_cast<uint16_t*>(rec + p.L.k_scale);
    uint16_t* kz_out = reinterpret_cast<uint16_t*>(rec + p.L.k_zero);
    uint16_t* kbs_out = reinterpret_cast<uint16_t*>(rec + p.L.kb_scale);
    if (kb < k) {
      // plane-B rows kb..k-1 carry no channel: zero codes and zero scales
      for (int i = tid; i < P * k; i += kQThreads) cB[i] = 0;
      for (int i = tid; i < n_groups * (k - kb); i += kQThreads)
        kbs_out[(i / (k - kb)) * k + kb + i % (k - kb)] = 0;
      __syncthreads();
    }
    for (int task = tid; task < n_groups * (kHeadDim / 2); task += kQThreads) {
      const int g = task / (kHeadDim / 2), c0 = 2 * (task % (kHeadDim / 2));
      const uint32_t* col = reinterpret_cast<const uint32_t*>(Ks + g * kKeyGroup * kHeadDim + c0);
      T2 lo = u32_as_pair(col[0], T()), hi = lo;
#pragma unroll 8
      for (int t = 1; t < kKeyGroup; ++t) {
        const T2 v = u32_as_pair(col[t * (kHeadDim / 2)], T());
        lo = __hmin2(lo, v);
        hi = __hmax2(hi, v);
      }
      const uint32_t lob = pair_as_u32(lo), hib = pair_as_u32(hi);
      float scale[2], rcp[2], zero[2];
      int qmax[2], j[2], pc[2], pj[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = c0 + e;
        j[e] = row_of[c];
        qmax[e] = j[e] >= 0 ? 15 : 3;
        pc[e] = key_pos(c);
        pj[e] = j[e] >= 0 ? boost_pos(j[e], k / 16) : 0;
        uint16_t sb, zb;
        scale[e] = quant_params<T>(bits_to_float(uint16_t(lob >> (16 * e)), T()),
                                   bits_to_float(uint16_t(hib >> (16 * e)), T()), qmax[e], sb, zb, zero[e]);
        rcp[e] = quant_rcp(scale[e]);
        // plane A of a boosted channel carries the high bits: scale 4*s4 (exact)
        const int pm = key_meta_pos(c);
        ks_out[g * kHeadDim + pm] = j[e] >= 0 ? exact_bits(4.0f * scale[e], T()) : sb;
        kz_out[g * kHeadDim + pm] = zb;
        if (j[e] >= 0) kbs_out[g * k + j[e]] = sb;
      }
      // codes of the group's 32 tokens; plane A gets code >> 2 for a boosted channel (its
      // low bits go to plane B) and the code itself otherwise; a channel that is not
      // boosted writes its "plane B" byte to a scratch row.  Elements within 2^-14 of a
      // rounding boundary (or of a group whose scale has no fast reciprocal) are redone
      // with the IEEE divide afterwards.
      uint8_t* a_base[2];
      uint8_t* b_base[2];
      int shift[2];
      bool all_exact[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        a_base[e] = cA + g * kKeyGroup * kHeadDim + pc[e];
        b_base[e] = j[e] >= 0 ? cB + g * kKeyGroup * k + pj[e] : cScratch;
        shift[e] = j[e] >= 0 ? 2 : 0;
        all_exact[e] = rcp[e] == 0.0f && scale[e] != 0.0f;
      }
      uint64_t redo = 0;
#pragma unroll 8
      for (int t = 0; t < kKeyGroup; ++t) {
        const uint32_t w = col[t * (kHeadDim / 2)];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          // the low byte of the bits is the code (the packing keeps two bits per byte)
          bool near;
          const uint32_t bits = quant_bits_fma(bits_to_float(uint16_t(w >> (16 * e)), T()), zero[e], rcp[e], near);
          redo |= uint64_t(near || all_exact[e]) << (2 * t + e);
          a_base[e][t * kHeadDim] = uint8_t(bits >> shift[e]);
          b_base[e][t * (j[e] >= 0 ? k : 0)] = uint8_t(bits);
        }
      }
      while (redo) {
        const int bit = __ffsll((long long)redo) - 1;
        redo &= redo - 1;
        const int t = bit >> 1, e = bit & 1;
        const uint32_t code = uint32_t(quant_code(bits_to_float(uint16_t(col[t * (kHeadDim / 2)] >> (16 * e)), T()),
                                                  zero[e], scale[e], qmax[e]));
        a_base[e][t * kHeadDim] = uint8_t(code >> shift[e]);
        b_base[e][t * (j[e] >= 0 ? k : 0)] = uint8_t(code);
      }
    }
  }

  // ---- a3: values, four tokens per warp (a quarter-warp each, 16 channels per lane)
  if (need_v) {
    using T2 = typename Pair<T>::type;
    const int warp = tid >> 5, lane = tid & 31, ql = lane & 7;
    uint16_t* vs_out = reinterpret_cast<uint16_t*>(rec + p.L.v_scale);
    uint16_t* vz_out = reinterpret_cast<uint16_t*>(rec + p.L.v_zero);
    for (int t0 = 4 * warp; t0 < P; t0 += 4 * (kQThreads / 32)) {
      const int t = t0 + (lane >> 3);
      const uint16_t* row = Vs + t * kHeadDim + 16 * ql;
      const uint4 r0 = lds128(row), r1 = lds128(row + 8);
      const uint32_t wv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
      T2 lo = u32_as_pair(wv[0], T()), hi = lo;
#pragma unroll
      for (int i = 1; i < 8; ++i) {
        lo = __hmin2(lo, u32_as_pair(wv[i], T()));
        hi = __hmax2(hi, u32_as_pair(wv[i], T()));
      }
      float mn = fminf(bits_to_float(uint16_t(pair_as_u32(lo)), T()), bits_to_float(uint16_t(pair_as_u32(lo) >> 16), T()));
      float mx = fmaxf(bits_to_float(uint16_t(pair_as_u32(hi)), T()), bits_to_float(uint16_t(pair_as_u32(hi) >> 16), T()));
#pragma unroll
      for (int off = 4; off > 0; off >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(kFull, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, off));
      }
      uint16_t sb, zb;
      float zero;
      const float scale = quant_params<T>(mn, mx, 3, sb, zb, zero);
      const float rcp = quant_rcp(scale);
      uint32_t packed[4] = {0u, 0u, 0u, 0u};
      bool redo = rcp == 0.0f && scale != 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float x = bits_to_float(uint16_t(wv[i >> 1] >> (16 * (i & 1))), T());
        bool near;
        packed[i >> 2] |= (quant_bits_fma(x, zero, rcp, near) & 0xffu) << (8 * (i & 3));
        redo |= near;
      }
      if (redo) {  // near a rounding boundary: the IEEE divide decides
#pragma unroll
        for (int i = 0; i < 4; ++i) packed[i] = 0u;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float x = bits_to_float(uint16_t(wv[i >> 1] >> (16 * (i & 1))), T());
          packed[i >> 2] |= uint32_t(quant_code(x, zero, scale, 3)) << (8 * (i & 3));
        }
      }
      *reinterpret_cast<uint4*>(cV + t * kHeadDim + 16 * ql) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      if (ql == 0) {
        vs_out[value_meta_pos(t)] = sb;
        vz_out[value_meta_pos(t)] = zb;
      }
    }
  }
  __syncthreads();

  // ---- pack the code planes into the record
  if (mode & kModeKeys) {
    uint32_t* kA = reinterpret_cast<uint32_t*>(rec + p.L.k_codes);
    for (int i = tid; i < P * (kHeadDim / 16); i += kQThreads) kA[i] = pack16(cA + 16 * i);
    const int kbw = k / 16;
    uint32_t* kB = reinterpret_cast<uint32_t*>(rec + p.L.kb_codes);
    for (int i = tid; i < P * kbw; i += kQThreads) kB[i] = pack16(cB + 16 * i);
  }
  if (need_v) {
    uint32_t* vq = reinterpret_cast<uint32_t*>(rec + p.L.v_codes);
    for (int i = tid; i < P * (kHeadDim / 16); i += kQThreads) {
      // value-code word i = ((2g + (m >> 2)) * 32 + 4w + q) * 4 + (m & 3): its element
      // e = 8a + 2b + f holds token 32g + 2q + 16a + 8(b >> 1) + f and channel
      // 16m + w + 8(b & 1), at bit elem_bit(e)
      const int mm = i & 3, ln = (i >> 2) & 31, blk = i >> 7;
      const uint8_t* base = cV + (32 * (blk >> 1) + 2 * (ln & 3)) * kHeadDim + 16 * (4 * (blk & 1) + mm) + (ln >> 2);
      uint32_t word = 0;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int a = e >> 3, b = (e >> 1) & 3, f = e & 1;
        word |= uint32_t(base[(16 * a + 8 * (b >> 1) + f) * kHeadDim + 8 * (b & 1)] & 3u) << elem_bit(e);
      }
      vq[i] = word;
    }
  }
  pdl_trigger();
}

// ------------------------------------------------------------------ residual window

// a4: append one token per sequence at position res_len[b], then res_len[b] += 1.
// One CTA per sequence; every head's K and V row is 256 bytes (16 x 16 bytes).
__global__ void __launch_bounds__(256) append_kernel(const uint4* k_new, const uint4* v_new, uint4* res_k,
                                                     uint4* res_v, int32_t* res_len, int Hkv, int P,
                                                     int32_t* err) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x;
  __shared__ int s_r;
  if (threadIdx.x == 0) s_r = res_len[b];
  __syncthreads();
  const int r = s_r;
  if (r < 0 || r >= P) {
    if (threadIdx.x == 0) flag_error(err, r >= P ? KVQ_DEV_ERR_RESIDUAL : KVQ_DEV_ERR_LENGTH);
    return;
  }
  const int n = Hkv * 16;
  for (int i = threadIdx.x; i < 2 * n; i += blockDim.x) {
    const int which = i / n, j = i % n, h = j >> 4, c = j & 15;
    const uint4* src = which ? v_new : k_new;
    uint4* dst = which ? res_v : res_k;
    dst[((size_t(b) * Hkv + h) * P + r) * 16 + c] = src[(size_t(b) * Hkv + h) * 16 + c];
  }
  __syncthreads();
  if (threadIdx.x == 0) res_len[b] = r + 1;
}

// a5 (second half): after the full windows were quantized into their new pages, link
// the pages and empty the windows.  Uses the same predicate as the quantize launch, so a
// sequence skipped there (bad page id, full table) is skipped here too.
__global__ void flush_commit_kernel(int32_t* res_len, const int32_t* new_page, int32_t* page_table,
                                    int max_pages, int32_t* num_pages, long long pool_pages, int batch,
                                    int P) {
  pdl_wait();
  pdl_trigger();
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < batch; b += gridDim.x * blockDim.x) {
    if (res_len[b] != P) continue;
    const int dst = new_page[b], np = num_pages[b];
    if (dst < 0 || np < 0 || np >= max_pages || dst >= pool_pages) continue;
    page_table[size_t(b) * max_pages + np] = dst;
    num_pages[b] = np + 1;
    res_len[b] = 0;
  }
}

// ------------------------------------------------------------------ host launchers

cudaError_t launch_quantize(const QuantParams& p, int n_items, int dtype, cudaStream_t stream) {
  if (n_items <= 0) return cudaSuccess;
  const size_t smem = QSmem::bytes(p.P, p.k, p.mode);
  // keys and values of a page in separate CTAs when both are requested
  const bool both = (p.mode & (kModeSelect | kModeKeys)) && (p.mode & kModeValues);
  const dim3 grid(n_items, p.Hkv, both ? 2 : 1);
  static int seen_bf16[64], seen_f16[64];
  if (dtype == KVQ_BF16) {
    const cudaError_t e = ensure_dynamic_smem(quantize_kernel<__nv_bfloat16>, int(smem), seen_bf16);
    if (e != cudaSuccess) return e;
    return launch_pdl(quantize_kernel<__nv_bfloat16>, grid, dim3(kQThreads), smem, stream, p);
  } else {
    const cudaError_t e = ensure_dynamic_smem(quantize_kernel<__half>, int(smem), seen_f16);
    if (e != cudaSuccess) return e;
    return launch_pdl(quantize_kernel<__half>, grid, dim3(kQThreads), smem, stream, p);
  }
}

cudaError_t launch_append(const void* k_new, const void* v_new, void* res_k, void* res_v, int32_t* res_len,
                          int batch, int Hkv, int P, int32_t* err, cudaStream_t stream) {
  if (batch <= 0) return cudaSuccess;
  return launch_pdl(append_kernel, dim3(batch), dim3(256), 0, stream, static_cast<const uint4*>(k_new),
                    static_cast<const uint4*>(v_new), static_cast<uint4*>(res_k), static_cast<uint4*>(res_v), res_len,
                    Hkv, P, err);
}

cudaError_t launch_flush_commit(int32_t* res_len, const int32_t* new_page, int32_t* page_table, int max_pages,
                                int32_t* num_pages, long long pool_pages, int batch, int P, cudaStream_t stream) {
  if (batch <= 0) return cudaSuccess;
  const int threads = 256, blocks = (batch + threads - 1) / threads;
  return launch_pdl(flush_commit_kernel, dim3(blocks), dim3(threads), 0, stream, res_len, new_page, page_table,
                    max_pages, num_pages, pool_pages, batch, P);
}

}  // namespace kvq
