// kvq_quantize.cu — page quantization (boost selection, two-plane keys, per-token
// values), residual append and residual flush for sm_100a.
//
// One CTA quantizes the keys of one (page, kv head) and another its values.  A CTA
// stages its [P][128] tile in shared memory with 16-byte asynchronous copies, then
//   a1  ranks channels by max |K| over the page (Kitty, Dynamic Channel-wise
//       Precision Boost; magnitude heuristic per the notes.yuuk.io wiki page), or by
//       w_c * (max - min) (MixKVQ summary, Abstract: query relevance times the
//       channel's quantization difficulty),
//   a2  quantizes every (key group, channel) asymmetrically — 4 bits for boosted
//       channels, split into a high plane and a low plane of 2-bit codes, 2 bits
//       otherwise (KIVI per-channel keys; Kitty two uniform 2-bit tensors),
//   a3  quantizes every token's values over the head dimension (KIVI per-token values),
// and writes the packed record.  Scales and zeros use explicit round-to-nearest fp32
// operations in the order the ABI documents, so codes, scales and zeros are
// bit-identical to any implementation of that definition.
//
// The codes never pass through shared memory: ldmatrix hands each lane the sixteen
// elements of one record word (the record's word order is the mma fragment order), the
// code of each element comes from two fused multiply-adds with the group's reciprocal
// bracketed from below and above (equal results prove the code; the rare element near
// a rounding boundary is redone with the IEEE divide), and byte permutes pack the codes.
#include "kvq_internal.cuh"

namespace kvq {

constexpr int kQThreads = 256;

// Tiles in shared memory: token t's 128 channels are 16 chunks of 16 bytes, chunk j
// stored at j ^ (t % 8), so the eight rows one ldmatrix matrix reads, or eight
// consecutive tokens read at one chunk, fall on eight different bank groups.
__device__ __forceinline__ uint32_t qtile_off(int t, int chunk) {
  return uint32_t(t) * 256u + (uint32_t(chunk ^ (t & 7)) << 4);
}

// Shared memory of one quantize CTA: the tile, then the code constants
// {-zero, r_lo, r_hi, scale} per (key group, channel) or per token, then (keys) the
// plane-B row of each channel, the channel of each plane-B row, the ranking keys and
// per-warp counts.
struct QSmem {
  __host__ __device__ static size_t tile(int P) { return size_t(P) * kHeadDim * 2; }
  static size_t key_bytes(int P) {
    return tile(P) + size_t(P / kKeyGroup) * kHeadDim * 16 + 2 * kHeadDim + kHeadDim * 4 + 8 * 4;
  }
  static size_t value_bytes(int P) { return tile(P) + size_t(P) * 16; }
  static size_t bytes(int P, int mode) {
    size_t b = 0;
    if (mode & (kModeSelect | kModeKeys)) b = key_bytes(P);
    if (mode & kModeValues) b = b > value_bytes(P) ? b : value_bytes(P);
    return b;
  }
};

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

// The definition: code = clamp(rint((x - zero) / scale), 0, qmax) in fp32.
__device__ __forceinline__ int quant_code(float x, float zero, float scale, int qmax) {
  if (scale == 0.0f) return 0;
  const float t = __fdiv_rn(__fsub_rn(x, zero), scale);
  float r = rintf(t);
  r = fminf(fmaxf(r, 0.0f), float(qmax));
  return int(r);
}

// Constants of the divide-free code of a group with scale s and zero z: {-z, r_lo,
// r_hi, s}.  r_lo and r_hi lie 8 units in the last place below and above the correctly
// rounded 1/s, so for d = x - z >= 0 the exact product d * r_lo is at most, and d * r_hi
// at least, the rounded quotient fl(d / s) (each of 1/s -> rcp and d / s -> fl loses at
// most 2^-24 relative; eight units are at least 8 * 2^-24).  Round-to-nearest-even is
// monotone, so when d * r_lo and d * r_hi round to the same integer, fl(d / s) rounds
// to it too: that is the code (the stored scale is rounded up, so no code exceeds qmax
// and the clamp never acts).  Scale 0 gives r_lo = r_hi = 0 (every code 0, as the
// definition gives); a scale whose reciprocal is not comfortably normal gives r_lo = 0,
// r_hi = inf, which sends every element of the group to the exact path.
__device__ __forceinline__ float4 code_consts(float zero, float scale) {
  float rlo, rhi;
  if (scale == 0.0f) {
    rlo = rhi = 0.0f;
  } else if (scale >= 0x1p-100f && scale <= 0x1p100f) {
    const uint32_t rb = __float_as_uint(__frcp_rn(scale));
    rlo = __uint_as_float(rb - 8u);
    rhi = __uint_as_float(rb + 8u);
  } else {
    rlo = 0.0f;
    rhi = __uint_as_float(0x7f800000u);
  }
  return make_float4(-zero, rlo, rhi, scale);
}

// x - zero in fp32 with one rounding for both 16-bit elements of a pair (PTX
// mixed-precision add: the 16-bit operand converts exactly, the sum rounds once).
__device__ __forceinline__ void sub_pair(uint32_t w, float nz0, float nz1, float& d0, float& d1, __half) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "add.rn.f32.f16 %0, l, %3;\n\tadd.rn.f32.f16 %1, h, %4;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "r"(w), "f"(nz0), "f"(nz1));
}
__device__ __forceinline__ void sub_pair(uint32_t w, float nz0, float nz1, float& d0, float& d1, __nv_bfloat16) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "add.rn.f32.bf16 %0, l, %3;\n\tadd.rn.f32.bf16 %1, h, %4;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "r"(w), "f"(nz0), "f"(nz1));
}

// Bits of fma(d, r, 1.5 * 2^23): for 0 <= d * r < 2^22 the result is 1.5 * 2^23 plus
// d * r rounded to the nearest integer (ties to even), so its low byte is that integer.
__device__ __forceinline__ uint32_t code_bits(float d, float r) {
  return __float_as_uint(__fmaf_rn(d, r, 12582912.0f));
}

// The code of one element whose two bracketed products rounded to different integers;
// k is the one from r_lo.  Inputs on the 16-bit grid often sit exactly on a rounding
// boundary (d = (k + 1/2) s): the rounded quotient is then exactly k + 1/2 and rint takes
// the even neighbour.  fma(-(k + 1/2), s, d) is the exact difference (one rounding of a
// value that is either 0 or far above the smallest subnormal), so it tells a tie apart
// without a divide; anything else is decided by the IEEE divide.
__device__ __forceinline__ uint32_t fix_code(float d, float x, float nz, float scale, uint32_t k, int qmax) {
  if (__fmaf_rn(-(float(k) + 0.5f), scale, d) == 0.0f) return k + (k & 1u);
  return uint32_t(quant_code(x, -nz, scale, qmax));
}

// Low bytes of four words -> one word, byte i from x_i.
__device__ __forceinline__ uint32_t low_bytes(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3) {
  return __byte_perm(__byte_perm(x0, x1, 0x0040), __byte_perm(x2, x3, 0x0040), 0x5410);
}

// Total order of fp32 scores as unsigned integers (larger score -> larger key).
__device__ __forceinline__ uint32_t order_key(float s) {
  const uint32_t u = __float_as_uint(__fadd_rn(s, 0.0f));  // -0 -> +0, like a float compare
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Quantizes the window or page tile of (item, kv head h) into record rec: the key part
// (z = 0) or the value part (z = gridDim.z - 1) of the requested modes.  last_k / last_v,
// when given, replace the tile's last token (the token an append-and-flush just wrote).
template <typename T, int P>
__device__ __forceinline__ void quantize_record(const QuantParams& p, int item, int h, uint8_t* rec,
                                                const uint16_t* last_k, const uint16_t* last_v) {
  const int tid = threadIdx.x;
  const int k = p.k;

  // z = 0: the key part of the requested modes, z = gridDim.z - 1: the value part
  const int kmodes = blockIdx.z == 0 ? p.mode & (kModeSelect | kModeKeys) : 0;
  const int mode = kmodes | (blockIdx.z == gridDim.z - 1 ? p.mode & kModeValues : 0);
  const bool need_k = kmodes != 0;
  const bool need_v = (mode & kModeValues) && !need_k;

  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t tile = smem_addr(smem);
  float4* qc = reinterpret_cast<float4*>(smem + QSmem::tile(P));  // keys [P/32][128], values [P]
  int8_t* row_of = reinterpret_cast<int8_t*>(qc + (P / kKeyGroup) * kHeadDim);  // plane-B row of a channel
  uint8_t* chan_of = reinterpret_cast<uint8_t*>(row_of + kHeadDim);             // channel of a plane-B row
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

  // ---- stage the tile (rows of 128 x 16-bit = 16 chunks of 16 bytes, swizzled)
  {
    const uint16_t* src = need_k ? p.k_src + item * p.k_page_stride + h * p.k_head_stride
                                 : p.v_src + item * p.v_page_stride + h * p.v_head_stride;
    const long long ts = need_k ? p.k_tok_stride : p.v_tok_stride;
    const uint16_t* last = need_k ? last_k : last_v;
    for (int i = tid; i < P * 16; i += kQThreads) {
      const int t = i >> 4, c = i & 15;
      const uint16_t* row = (last && t == P - 1) ? last : src + t * ts;
      cp_async16(smem + qtile_off(t, c), row + c * 8, 16);
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;

  if (need_k) {
    using T2 = typename Pair<T>::type;
    const int NG = P / kKeyGroup;
    // ---- exact min / max per (key group, channel pair), packed pairs (exact)
    const int g1 = tid >> 6, c0 = 2 * (tid & 63);
    const bool has_pair = g1 < NG;
    uint32_t lob = 0, hib = 0;
    uint32_t* mm = reinterpret_cast<uint32_t*>(qc);  // scratch [NG][min, max][64 pairs]
    if (has_pair) {
      const uint8_t* base = smem + (c0 & 7) * 2;
      const int t0 = g1 * kKeyGroup;
      T2 lo = u32_as_pair(lds32(base + qtile_off(t0, c0 >> 3)), T()), hi = lo;
#pragma unroll 8
      for (int t = 1; t < kKeyGroup; ++t) {
        const T2 v = u32_as_pair(lds32(base + qtile_off(t0 + t, c0 >> 3)), T());
        lo = __hmin2(lo, v);
        hi = __hmax2(hi, v);
      }
      lob = pair_as_u32(lo);
      hib = pair_as_u32(hi);
      if (mode & kModeSelect) {
        mm[(2 * g1) * 64 + (tid & 63)] = lob;
        mm[(2 * g1 + 1) * 64 + (tid & 63)] = hib;
      }
    }
    __syncthreads();

    // ---- a1: boosted channels (or read them back from the record)
    if (mode & kModeSelect) {
      uint32_t* keys = reinterpret_cast<uint32_t*>(chan_of + kHeadDim);  // [128]
      int* warp_cnt = reinterpret_cast<int*>(keys + kHeadDim);           // [8]
      if (tid < kHeadDim) {
        // score from the page's exact min / max: max(|min|, |max|) (magnitude) or
        // w * (max - min) (query-aware)
        const int c = tid;
        float mn = __int_as_float(0x7f800000), mx = -mn;
        for (int g = 0; g < NG; ++g) {
          mn = fminf(mn, bits_to_float(uint16_t(mm[(2 * g) * 64 + (c >> 1)] >> (16 * (c & 1))), T()));
          mx = fmaxf(mx, bits_to_float(uint16_t(mm[(2 * g + 1) * 64 + (c >> 1)] >> (16 * (c & 1))), T()));
        }
        // A magnitude is a 16-bit value widened to fp32, so its 13 low bits are zero:
        // the channel index fills them and every key is unique (ties to the lower index).
        keys[c] = p.qw ? order_key(__fmul_rn(p.qw[h * kHeadDim + c], __fsub_rn(mx, mn)))
                       : (__float_as_uint(__fadd_rn(fmaxf(fabsf(mn), fabsf(mx)), 0.0f)) | uint32_t(127 - c));
      }
      __syncthreads();
      // rank of channel c: channels ahead of it, two threads per channel (64 each)
      const int c = tid >> 1, half = tid & 1;
      const uint32_t kc = keys[c];
      int rank = 0;
      if (!p.qw) {
#pragma unroll 4
        for (int i = 0; i < 64; i += 4) {
          const uint4 v = *reinterpret_cast<const uint4*>(keys + 64 * half + i);
          rank += int(v.x > kc) + int(v.y > kc) + int(v.z > kc) + int(v.w > kc);
        }
      } else {
#pragma unroll 8
        for (int i = 0; i < 64; ++i) {
          const int o = 64 * half + i;
          const uint32_t ko = keys[o];
          rank += int(ko > kc || (ko == kc && o < c));
        }
      }
      rank += __shfl_xor_sync(kFull, rank, 1);
      const bool boosted = rank < kb;
      // plane-B row of a boosted channel: boosted channels with a lower index before it
      const unsigned ballot = __ballot_sync(kFull, boosted && half == 0);
      if (lane == 0) warp_cnt[warp] = __popc(ballot);
      __syncthreads();
      if (half == 0) {
        int before = 0;
        for (int w = 0; w < warp; ++w) before += warp_cnt[w];
        const int row = boosted ? before + __popc(ballot & ((1u << lane) - 1u)) : -1;
        row_of[c] = int8_t(row);
        if (row >= 0) {
          rec[p.L.boost_idx + row] = uint8_t(c);
          chan_of[row] = uint8_t(c);
        }
      }
      if (tid >= kb && tid < k) {  // unused rows
        rec[p.L.boost_idx + tid] = 0;
        chan_of[tid] = 0xff;
      }
    } else {
      if (tid < kHeadDim) row_of[tid] = -1;
      __syncthreads();
      if (tid < k) {
        const int c = tid < kb ? rec[p.L.boost_idx + tid] : 0xff;
        chan_of[tid] = uint8_t(c < kHeadDim ? c : 0xff);
        if (c < kHeadDim) row_of[c] = int8_t(tid);
      }
    }
    __syncthreads();

    if (mode & kModeKeys) {
      uint16_t* ks_out = reinterpret_cast<uint16_t*>(rec + p.L.k_scale);
      uint16_t* kz_out = reinterpret_cast<uint16_t*>(rec + p.L.k_zero);
      uint16_t* kbs_out = reinterpret_cast<uint16_t*>(rec + p.L.kb_scale);
      // ---- a2 constants: one thread per (group, channel pair), min / max still in registers
      for (int i = tid; i < NG * (k - kb); i += kQThreads)  // rows kb..k-1 carry no channel
        kbs_out[(i / (k - kb)) * k + kb + i % (k - kb)] = 0;
      if (has_pair) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = c0 + e, j = row_of[c];
          uint16_t sb, zb;
          float zero;
          const float scale = quant_params<T>(bits_to_float(uint16_t(lob >> (16 * e)), T()),
                                              bits_to_float(uint16_t(hib >> (16 * e)), T()), j >= 0 ? 15 : 3, sb,
                                              zb, zero);
          // plane A of a boosted channel carries the high bits: scale 4*s4 (exact)
          const int pm = key_meta_pos(c);
          ks_out[g1 * kHeadDim + pm] = j >= 0 ? exact_bits(4.0f * scale, T()) : sb;
          kz_out[g1 * kHeadDim + pm] = zb;
          if (j >= 0) kbs_out[g1 * k + j] = sb;
          qc[g1 * kHeadDim + c] = code_consts(zero, scale);
        }
      }
      __syncthreads();

      // ---- a2 plane A (and plane B when every channel is boosted: row j = channel j).
      // Warp -> (group g, word half hh), 4 tokens per step; lane -> token tbase + lane / 8,
      // word half a = (lane / 4) % 2, q = lane % 4.  Its eight elements are channels
      // c(j, f) = 64hh + 32a + 8j + 2q + f, which sit at element 8a + 2j + f of record
      // word 2q + hh of the token; the partner lane (a ^ 1) holds the other eight.
      {
        const bool all_b = kb == kHeadDim;
        const int per = P / 16;
        const int it0 = warp * per;
        const int g = it0 >> 4, hh = (it0 >> 3) & 1;
        const int a = (lane >> 2) & 1, q = lane & 3;
        float nz[8], rlo[8], rhi[8];
        uint32_t bm[2] = {0u, 0u};  // byte j = 0x3f where channel c(j, f) is boosted
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int f = 0; f < 2; ++f) {
            const int c = 64 * hh + 32 * a + 8 * j + 2 * q + f;
            const float4 v = qc[g * kHeadDim + c];
            nz[2 * j + f] = v.x;
            rlo[2 * j + f] = v.y;
            rhi[2 * j + f] = v.z;
            if (row_of[c] >= 0) bm[f] |= 0x3fu << (8 * j);
          }
        // ldmatrix: lane L gives row L % 8 of matrix L / 8 = j: token offset (L % 8) / 2,
        // half (L % 8) % 2, chunk 8hh + 4 * half + j
        const int rho = lane & 7;
        const int chunk = 8 * hh + 4 * (rho & 1) + (lane >> 3);
        uint32_t* kA = reinterpret_cast<uint32_t*>(rec + p.L.k_codes);
        uint32_t* kB = reinterpret_cast<uint32_t*>(rec + p.L.kb_codes);
        for (int it = 0; it < per; ++it) {
          const int tbase = 32 * g + 4 * ((it0 + it) & 7);
          uint32_t x[4];
          ldmatrix_x4(x, tile + qtile_off(tbase + (rho >> 1), chunk));
          uint32_t lo[8], acc = 0u;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float d0, d1;
            sub_pair(x[j], nz[2 * j], nz[2 * j + 1], d0, d1, T());
            lo[2 * j] = code_bits(d0, rlo[2 * j]);
            lo[2 * j + 1] = code_bits(d1, rlo[2 * j + 1]);
            acc |= (lo[2 * j] ^ code_bits(d0, rhi[2 * j])) | (lo[2 * j + 1] ^ code_bits(d1, rhi[2 * j + 1]));
          }
          uint32_t X0 = low_bytes(lo[0], lo[2], lo[4], lo[6]);  // element 8a + 2j, byte j
          uint32_t X1 = low_bytes(lo[1], lo[3], lo[5], lo[7]);  // element 8a + 2j + 1
          if (acc != 0u) {  // an element near a rounding boundary
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
              for (int f = 0; f < 2; ++f) {
                uint32_t& X = f ? X1 : X0;
                const float xv = bits_to_float(uint16_t(x[j] >> (16 * f)), T());
                const float d = __fadd_rn(xv, nz[2 * j + f]);
                const uint32_t k0 = (X >> (8 * j)) & 0xffu;
                if (code_bits(d, rhi[2 * j + f]) != 0x4B400000u + k0) {
                  const int c = 64 * hh + 32 * a + 8 * j + 2 * q + f;
                  const uint32_t code = fix_code(d, xv, nz[2 * j + f], qc[g * kHeadDim + c].w, k0,
                                                 ((bm[f] >> (8 * j)) & 1u) ? 15 : 3);
                  X = (X & ~(0xffu << (8 * j))) | (code << (8 * j));
                }
              }
          }
          // plane A: the code, or its high bits where the channel is boosted
          const uint32_t A0 = (((X0 >> 2) & bm[0]) | (X0 & ~bm[0])) & 0x03030303u;
          const uint32_t A1 = (((X1 >> 2) & bm[1]) | (X1 & ~bm[1])) & 0x03030303u;
          const uint32_t wa = A0 + 16u * A1;
          const uint32_t wa_other = __shfl_xor_sync(kFull, wa, 4);
          const int t = tbase + (lane >> 3);
          if (a == 0) kA[t * 8 + 2 * q + hh] = wa + 4u * wa_other;
          if (all_b) {
            const uint32_t wb = (X0 & 0x03030303u) + 16u * (X1 & 0x03030303u);
            const uint32_t wb_other = __shfl_xor_sync(kFull, wb, 4);
            if (a == 0) kB[t * 8 + 2 * q + hh] = wb + 4u * wb_other;
          }
        }
      }

      // ---- a2 plane B: the low bits of the boosted channels.  Task = (4 tokens of one
      // group, plane-B word wb); its sixteen elements are rows j = 16s + 8r + 2q + f at
      // word position 4(k/16)q + 4s + 2r + f - 16wb, gathered from their channels.
      if (k > 0 && kb < kHeadDim) {
        const int KW = k / 16;
        const int n_tasks = KW * P / 4;
        uint32_t* kB = reinterpret_cast<uint32_t*>(rec + p.L.kb_codes);
        const int lg = 31 - __clz(4 * KW);  // log2(4 KW)
        for (int task = tid; task < n_tasks; task += kQThreads) {
          const int wb = task & (KW - 1), t0 = 4 * (task / KW), g = t0 >> 5;
          uint32_t word[4] = {0u, 0u, 0u, 0u};
#pragma unroll 1
          for (int a = 0; a < 2; ++a) {
            uint32_t co[8];
            float nz[8], rlo[8], rhi[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {  // element e = 8a + i
              const int pos = 16 * wb + 8 * a + i;
              const int q = pos >> lg, rem = pos & ((1 << lg) - 1);
              const int j = 16 * (rem >> 2) + 8 * ((rem >> 1) & 1) + 2 * q + (rem & 1);
              const int c = chan_of[j];
              if (c < kHeadDim) {
                const float4 v = qc[g * kHeadDim + c];
                nz[i] = v.x;
                rlo[i] = v.y;
                rhi[i] = v.z;
                co[i] = uint32_t((c >> 3) << 4 | (c & 7) << 1);
              } else {  // no channel: code 0 (r_lo = r_hi = 0 never needs the fallback)
                nz[i] = rlo[i] = rhi[i] = 0.0f;
                co[i] = 0u;
              }
            }
#pragma unroll
            for (int n = 0; n < 4; ++n) {
              const int t = t0 + n;
              const uint32_t sw = uint32_t(t & 7) << 4;
              uint32_t lo[8], xp[4], acc = 0u;
#pragma unroll
              for (int i = 0; i < 8; i += 2) {
                const uint32_t xl = *reinterpret_cast<const uint16_t*>(smem + t * 256 + (co[i] ^ sw));
                const uint32_t xh = *reinterpret_cast<const uint16_t*>(smem + t * 256 + (co[i + 1] ^ sw));
                xp[i >> 1] = xl | (xh << 16);
                float d0, d1;
                sub_pair(xp[i >> 1], nz[i], nz[i + 1], d0, d1, T());
                lo[i] = code_bits(d0, rlo[i]);
                lo[i + 1] = code_bits(d1, rlo[i + 1]);
                acc |= (lo[i] ^ code_bits(d0, rhi[i])) | (lo[i + 1] ^ code_bits(d1, rhi[i + 1]));
              }
              uint32_t X0 = low_bytes(lo[0], lo[2], lo[4], lo[6]);
              uint32_t X1 = low_bytes(lo[1], lo[3], lo[5], lo[7]);
              if (acc != 0u) {  // an element near a rounding boundary
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  uint32_t& X = (i & 1) ? X1 : X0;
                  const int sh = 8 * (i >> 1);
                  const float xv = bits_to_float(uint16_t(xp[i >> 1] >> (16 * (i & 1))), T());
                  const float d = __fadd_rn(xv, nz[i]);
                  const uint32_t k0 = (X >> sh) & 0xffu;
                  if (code_bits(d, rhi[i]) != 0x4B400000u + k0) {
                    const int c = int((co[i] >> 4) << 3 | ((co[i] >> 1) & 7u));
                    X = (X & ~(0xffu << sh)) | (fix_code(d, xv, nz[i], qc[g * kHeadDim + c].w, k0, 15) << sh);
                  }
                }
              }
              // element 8a + 2b + f at bit 8b + 4f + 2a
              word[n] |= ((X0 & 0x03030303u) + 16u * (X1 & 0x03030303u)) << (2 * a);
            }
          }
#pragma unroll
          for (int n = 0; n < 4; ++n) kB[(t0 + n) * KW + wb] = word[n];
        }
      }
    }
  }

  if (need_v) {
    using T2 = typename Pair<T>::type;
    uint16_t* vs_out = reinterpret_cast<uint16_t*>(rec + p.L.v_scale);
    uint16_t* vz_out = reinterpret_cast<uint16_t*>(rec + p.L.v_zero);
    // ---- a3 constants: two threads per token (64 channels each), packed min / max
    {
      const int t = tid >> 1, hf = tid & 1;
      if (t < P) {  // whole warps
        T2 lo, hi;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = lds128(smem + qtile_off(t, 8 * hf + ((i + 4 * hf) & 7)));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int n = 0; n < 4; ++n) {
            const T2 x = u32_as_pair(w[n], T());
            if (i == 0 && n == 0) {
              lo = hi = x;
            } else {
              lo = __hmin2(lo, x);
              hi = __hmax2(hi, x);
            }
          }
        }
        float mn = fminf(bits_to_float(uint16_t(pair_as_u32(lo)), T()), bits_to_float(uint16_t(pair_as_u32(lo) >> 16), T()));
        float mx = fmaxf(bits_to_float(uint16_t(pair_as_u32(hi)), T()), bits_to_float(uint16_t(pair_as_u32(hi) >> 16), T()));
        mn = fminf(mn, __shfl_xor_sync(kFull, mn, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        if (hf == 0) {
          uint16_t sb, zb;
          float zero;
          const float scale = quant_params<T>(mn, mx, 3, sb, zb, zero);
          vs_out[value_meta_pos(t)] = sb;
          vz_out[value_meta_pos(t)] = zb;
          qc[t] = code_consts(zero, scale);
        }
      }
    }
    __syncthreads();

    // ---- a3 codes.  Warp -> group g and P/32 consecutive channel blocks m; lane (w, q)
    // builds record word ((2g + m/4) * 32 + lane) * 4 + m % 4, whose element
    // e = 8a + 2b + f (b = 2u + v) is token 32g + 16a + 8u + 2q + f, channel 16m + 8v + w:
    // exactly what ldmatrix.trans of the matrices (a, u, v) hands this lane.
    {
      const int NT = P / 32;
      const int task0 = warp * NT, g = task0 >> 3;
      const int q = lane & 3;
      float nz[8], rlo[8], rhi[8];  // token (a, u, f) at index 4a + 2u + f
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int t = 32 * g + 16 * (i >> 2) + 8 * ((i >> 1) & 1) + 2 * q + (i & 1);
        const float4 v = qc[t];
        nz[i] = v.x;
        rlo[i] = v.y;
        rhi[i] = v.z;
      }
      const int mi = lane >> 3, rho = lane & 7;
      uint32_t* vq = reinterpret_cast<uint32_t*>(rec + p.L.v_codes) +
                     ((2 * g + ((task0 & 7) >> 2)) * 32 + lane) * 4 + (task0 & 3);
#pragma unroll 1
      for (int n = 0; n < NT; ++n) {
        const int m = (task0 + n) & 7;
        uint32_t word = 0u, acc = 0u;
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          uint32_t x[4];
          ldmatrix_x4_trans(x, tile + qtile_off(32 * g + 16 * a + 8 * (mi >> 1) + rho, 2 * m + (mi & 1)));
          uint32_t lo[8];
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int ti = 4 * a + 2 * (b >> 1);
            float d0, d1;
            sub_pair(x[b], nz[ti], nz[ti + 1], d0, d1, T());
            lo[2 * b] = code_bits(d0, rlo[ti]);
            lo[2 * b + 1] = code_bits(d1, rlo[ti + 1]);
            acc |= (lo[2 * b] ^ code_bits(d0, rhi[ti])) | (lo[2 * b + 1] ^ code_bits(d1, rhi[ti + 1]));
          }
          const uint32_t X0 = low_bytes(lo[0], lo[2], lo[4], lo[6]) & 0x03030303u;
          const uint32_t X1 = low_bytes(lo[1], lo[3], lo[5], lo[7]) & 0x03030303u;
          word += (X0 + 16u * X1) << (2 * a);
        }
        // Near a rounding boundary the IEEE divide decides.  The fragments are loaded again
        // by the whole warp (ldmatrix is a warp-wide instruction and must not run in a
        // branch that only some lanes take); the lanes that need it rebuild their word.
        if (__any_sync(kFull, acc != 0u)) {
          const bool redo = acc != 0u;
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            uint32_t x[4];
            ldmatrix_x4_trans(x, tile + qtile_off(32 * g + 16 * a + 8 * (mi >> 1) + rho, 2 * m + (mi & 1)));
            if (redo) {
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int b = i >> 1, f = i & 1, ti = 4 * a + 2 * (b >> 1) + f, sh = elem_bit(8 * a + i);
                const float xv = bits_to_float(uint16_t(x[b] >> (16 * f)), T());
                const float d = __fadd_rn(xv, nz[ti]);
                const uint32_t k0 = (word >> sh) & 3u;
                if (code_bits(d, rhi[ti]) != 0x4B400000u + k0) {
                  const int t = 32 * g + 16 * a + 8 * (b >> 1) + 2 * q + f;
                  const uint32_t code = fix_code(d, xv, nz[ti], qc[t].w, k0, 3);
                  word = (word & ~(3u << sh)) | (code << sh);
                }
              }
            }
          }
        }
        vq[n] = word;
      }
    }
  }
}

// Modes: quantize pages (dst_pages), flush full windows (flush), or append-and-flush
// (append: a4 + a5 in one launch).  In the last, every CTA of sequence `item` appends its
// row of the new token (z = 0: keys, z = 1: values of kv head h) at position res_len of
// the window, and when the window is then full quantizes its part of the window into the
// page new_page reserves.  The last of the sequence's 2 * Hkv CTAs to arrive writes the
// lengths and the page-table entry, so every CTA has read the old length before it
// changes.  The outcome, error bits included, is that of kvq_append_token followed by
// kvq_flush_residual.
// P (page tokens: 32, 64 or 128) is a template parameter so that every trip count, group
// count and tile offset is a constant.
template <typename T, int P>
__global__ void __launch_bounds__(kQThreads, 4) quantize_kernel(const __grid_constant__ QuantParams p) {
  pdl_wait();
  const int item = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  int dst = -1, np = 0, r = 0;
  bool go = false, app = false;
  const uint16_t* last = nullptr;
  if (p.append) {
    // the next kernel may be scheduled now: it reads nothing of ours before its own wait
    pdl_trigger();
    const bool first = h == 0 && blockIdx.z == 0;
    r = p.res_len_w[item];
    if (r < 0 || r > P) {  // the append flags it; the flush skips a window that is not full
      if (first && tid == 0) flag_error(p.err, r > P ? KVQ_DEV_ERR_RESIDUAL : KVQ_DEV_ERR_LENGTH);
      return;
    }
    app = r < P;  // r == P: a full window left by an earlier skipped flush
    if (!app && first && tid == 0) flag_error(p.err, KVQ_DEV_ERR_RESIDUAL);
    const size_t hrow = size_t(item) * p.Hkv + h;
    const uint16_t* src = (blockIdx.z == 0 ? p.k_new : p.v_new) + hrow * kHeadDim;
    if (app && tid < 16)
      reinterpret_cast<uint4*>(blockIdx.z == 0 ? p.res_k : p.res_v)[(hrow * P + r) * 16 + tid] =
          reinterpret_cast<const uint4*>(src)[tid];
    if (!app || r + 1 == P) {
      dst = p.dst_pages[item];
      np = p.num_pages_w[item];
      if (dst < 0 || np < 0 || np >= p.max_pages) {
        if (first && tid == 0) flag_error(p.err, KVQ_DEV_ERR_TABLE_FULL);
      } else if (dst >= p.pool_pages) {
        if (tid == 0) flag_error(p.err, KVQ_DEV_ERR_PAGE_RANGE);
      } else {
        go = true;
        if (app) last = src;  // the token just appended, read from its source
      }
    }
  } else {
    if (p.flush) {
      if (p.res_len[item] != P) return;
      dst = p.dst_pages[item];
      np = p.num_pages[item];
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
    go = true;
  }
  if (go) quantize_record<T, P>(p, item, h, p.pool + (size_t(dst) * p.Hkv + h) * p.L.record, last, last);
  if (p.append) {
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const int n = atomicAdd(p.counters + item, 1);
      if (n == int(gridDim.y * gridDim.z) - 1) {
        p.counters[item] = 0;
        if (go) {
          p.page_table[size_t(item) * p.max_pages + np] = dst;
          p.num_pages_w[item] = np + 1;
          p.res_len_w[item] = 0;
        } else if (app) {
          p.res_len_w[item] = r + 1;
        }
      }
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

template <typename T, int P>
static cudaError_t launch_quantize_p(const QuantParams& p, dim3 grid, size_t smem, cudaStream_t stream) {
  static int seen[64];
  const cudaError_t e = ensure_dynamic_smem(quantize_kernel<T, P>, int(smem), seen);
  if (e != cudaSuccess) return e;
  return launch_pdl(quantize_kernel<T, P>, grid, dim3(kQThreads), smem, stream, p);
}

template <typename T>
static cudaError_t launch_quantize_t(const QuantParams& p, dim3 grid, size_t smem, cudaStream_t stream) {
  switch (p.P) {
    case 32: return launch_quantize_p<T, 32>(p, grid, smem, stream);
    case 64: return launch_quantize_p<T, 64>(p, grid, smem, stream);
    case 128: return launch_quantize_p<T, 128>(p, grid, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_quantize(const QuantParams& p, int n_items, int dtype, cudaStream_t stream) {
  if (n_items <= 0) return cudaSuccess;
  const size_t smem = QSmem::bytes(p.P, p.mode);
  // keys and values of a page in separate CTAs when both are requested
  const bool both = (p.mode & (kModeSelect | kModeKeys)) && (p.mode & kModeValues);
  const dim3 grid(n_items, p.Hkv, both ? 2 : 1);
  return dtype == KVQ_BF16 ? launch_quantize_t<__nv_bfloat16>(p, grid, smem, stream)
                           : launch_quantize_t<__half>(p, grid, smem, stream);
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
