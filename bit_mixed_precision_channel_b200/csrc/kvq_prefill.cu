// kvq_prefill.cu — prefill attention with cumulative attention scores, token retention
// and the gather of the kept tokens (sm_100a).
//
// MiniKV summary (f-binder), "proposed method": the prompt is processed at prefill, the
// tokens to keep are chosen by their cumulative attention score (heavy hitters) together
// with a recent window, and a two-stage selective flash-attention kernel returns the
// attention output and those scores in linear memory.  Here:
//   pass 1 (prefill_fwd)   causal flash attention, one CTA per (64 query rows, query
//                          head): the output rows and each row's log2-sum-exp;
//   pass 2 (prefill_score) one CTA per (64 key rows, KV head): recomputes K Q^T for the
//                          query blocks at or after the key block and the query heads of
//                          the KV head, turns it into probabilities with the rows'
//                          log2-sum-exp, and sums them per key — no L x L matrix is kept;
//   retain_kernel          per KV head: the last n_recent positions plus the n_heavy
//                          best-scored others (radix select on the fp32 scores, ties to the
//                          lower position), ascending;
//   gather_kernel          the kept tokens of every KV head, compacted token-major, ready
//                          for the page quantizer.
// Products run on the tensor cores (mma.sync m16n8k16, fp32 accumulate) with operands
// in the cache dtype; fp16 probabilities carry 11 bits, bf16 ones are split into a high
// and a low bf16 part.
#include "kvq_internal.cuh"

namespace kvq {
namespace pf {

constexpr int kRows = 64;  // query rows (pass 1) or key rows (pass 2) per CTA
constexpr int kThreads = 128;
constexpr int kTile = kRows * 256;  // one [64][128] tile of the 16-bit dtype

// Byte offset of 16-byte chunk c (0..15) of row r in a [rows][256 B] tile: the chunk
// index is XOR-ed with r % 8, so that the eight rows an ldmatrix reads at one chunk
// column fall into different banks.
__device__ __forceinline__ uint32_t swz(int r, int c) { return uint32_t(r * 256 + ((c ^ (r & 7)) << 4)); }

// Copies rows [0, valid) of a 64-row tile (row i at src + i * stride elements) into
// shared memory with cp.async; rows at or past `valid` are zero-filled.
__device__ __forceinline__ void load_tile(uint8_t* dst, const uint16_t* src, long long stride, int valid, int tid) {
#pragma unroll
  for (int i = tid; i < kRows * 16; i += kThreads) {
    const int r = i >> 4, c = i & 15;
    const bool ok = r < valid;
    cp_async16(dst + swz(r, c), src + (ok ? r : 0) * stride + c * 8, ok ? 16u : 0u);
  }
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// A fragments (row-major 16 x 16) of rows r0 .. r0 + 15 of a tile, k-step ks.
__device__ __forceinline__ void ld_a(uint32_t (&a)[4], const uint8_t* tile, int r0, int ks, int lane) {
  const int mi = lane >> 3, r = lane & 7;
  ldmatrix_x4(a, smem_addr(tile + swz(r0 + ((mi & 1) ? 8 : 0) + r, 2 * ks + (mi >> 1))));
}
// B fragments (k = channels, n = tile rows) of n-tiles (n0 .. n0 + 7) and (n0 + 8 .. n0 + 15), k-step ks:
// b[0], b[1] for the first n-tile, b[2], b[3] for the second.
__device__ __forceinline__ void ld_b_rows(uint32_t (&b)[4], const uint8_t* tile, int n0, int ks, int lane) {
  const int mi = lane >> 3, r = lane & 7;
  ldmatrix_x4(b, smem_addr(tile + swz(n0 + ((mi >> 1) ? 8 : 0) + r, 2 * ks + (mi & 1))));
}
// B fragments (k = tile rows, n = channels) of the k-step of rows k0 .. k0 + 15 and the
// channel n-tiles (c0 .. c0 + 7), (c0 + 8 .. c0 + 15): b[0], b[1] and b[2], b[3].
__device__ __forceinline__ void ld_b_trans(uint32_t (&b)[4], const uint8_t* tile, int k0, int c0, int lane) {
  const int mi = lane >> 3, r = lane & 7;
  ldmatrix_x4_trans(b, smem_addr(tile + swz(k0 + ((mi & 1) ? 8 : 0) + r, (c0 >> 3) + (mi >> 1))));
}

// Two floats as a pair of the 16-bit type (low half = a).
__device__ __forceinline__ uint32_t pk(float a, float b, __half) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(b), "f"(a));
  return d;
}
__device__ __forceinline__ uint32_t pk(float a, float b, __nv_bfloat16) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(b), "f"(a));
  return d;
}
__device__ __forceinline__ float2 upk(uint32_t u, __half) { return __half22float2(u32_as_h2(u)); }
__device__ __forceinline__ float2 upk(uint32_t u, __nv_bfloat16) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

struct PrefillParams {
  const uint16_t* q;  // [L][Hq][128]
  const uint16_t* k;  // [L][Hkv][128]
  const uint16_t* v;
  int L, Hq, Hkv, gqa;
  float c_log2;       // sm_scale * log2(e)
  float* out;         // [L][Hq][128]
  float* lse;         // [Hq][L]: log2-sum-exp of every row (log2 units)
  float* score;       // [Hkv][L]
};

// ---------------------------------------------------------------- pass 1

template <typename T>
__global__ void __launch_bounds__(kThreads) prefill_fwd(const __grid_constant__ PrefillParams p) {
  extern __shared__ __align__(128) uint8_t smem[];  // Q tile | 2 x (K tile, V tile)
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, qd = lane & 3;
  const int qb = gridDim.x - 1 - blockIdx.x;  // the longest rows first
  const int h = blockIdx.y, kvh = h / p.gqa;
  const int q0 = qb * kRows;
  const long long qs = (long long)p.Hq * 128, ks_ = (long long)p.Hkv * 128;
  uint8_t* Qt = smem;
  load_tile(Qt, p.q + (long long)q0 * qs + h * 128, qs, min(kRows, p.L - q0), tid);
  load_tile(smem + kTile, p.k + kvh * 128, ks_, min(kRows, p.L), tid);
  load_tile(smem + 2 * kTile, p.v + kvh * 128, ks_, min(kRows, p.L), tid);
  cp_commit();

  uint32_t qa[8][4];
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) o[i][j] = 0.0f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.0f, 0.0f};
  const int r0 = warp * 16;  // this warp's rows in the tile
  const int row_g = q0 + r0 + g, row_g8 = row_g + 8;

  for (int kb = 0; kb <= qb; ++kb) {
    uint8_t* Kt = smem + kTile + (kb & 1) * 2 * kTile;
    uint8_t* Vt = Kt + kTile;
    if (kb < qb) {
      uint8_t* Kn = smem + kTile + ((kb + 1) & 1) * 2 * kTile;
      const int k0 = (kb + 1) * kRows;
      load_tile(Kn, p.k + (long long)k0 * ks_ + kvh * 128, ks_, min(kRows, p.L - k0), tid);
      load_tile(Kn + kTile, p.v + (long long)k0 * ks_ + kvh * 128, ks_, min(kRows, p.L - k0), tid);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    if (kb == 0) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) ld_a(qa[ks], Qt, r0, ks, lane);
    }
    // S = Q K^T: 16 rows x 64 keys per warp
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) s[i][j] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b[4];
        ld_b_rows(b, Kt, 16 * np, ks, lane);
        mma_16816(s[2 * np], qa[ks], b[0], b[1], T());
        mma_16816(s[2 * np + 1], qa[ks], b[2], b[3], T());
      }
    // scale, causal mask and the key range
    const int key0 = kb * kRows;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int key = key0 + 8 * nt + 2 * qd + (j & 1);
        const int row = (j >> 1) ? row_g8 : row_g;
        const float x = (key <= row && key < p.L) ? s[nt][j] * p.c_log2 : -INFINITY;
        s[nt][j] = x;
        mx[j >> 1] = fmaxf(mx[j >> 1], x);
      }
    float alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(kFull, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(kFull, mx[r], 2));
      const float mn = fmaxf(m[r], mx[r]);
      alpha[r] = mn == -INFINITY ? 1.0f : ex2(m[r] - mn);
      m[r] = mn;
      l[r] *= alpha[r];
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      o[i][0] *= alpha[0];
      o[i][1] *= alpha[0];
      o[i][2] *= alpha[1];
      o[i][3] *= alpha[1];
    }
    // probabilities -> A fragments of the PV product (S accumulators of n-tiles 2ks and
    // 2ks + 1 form the A fragment of k-step ks)
    uint32_t pa[4][4], pl[4][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      float pv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float mm = m[j >> 1];
        pv[j] = mm == -INFINITY ? 0.0f : ex2(s[nt][j] - mm);
        l[j >> 1] += pv[j];
      }
      const int ks = nt >> 1, hi = nt & 1;
      pa[ks][2 * hi] = pk(pv[0], pv[1], T());
      pa[ks][2 * hi + 1] = pk(pv[2], pv[3], T());
      if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        const float2 h0 = upk(pa[ks][2 * hi], T()), h1 = upk(pa[ks][2 * hi + 1], T());
        pl[ks][2 * hi] = pk(pv[0] - h0.x, pv[1] - h0.y, T());
        pl[ks][2 * hi + 1] = pk(pv[2] - h1.x, pv[3] - h1.y, T());
      }
    }
    // O += P V: 16 rows x 128 channels per warp
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int cp = 0; cp < 8; ++cp) {
        uint32_t b[4];
        ld_b_trans(b, Vt, 16 * ks, 16 * cp, lane);
        mma_16816(o[2 * cp], pa[ks], b[0], b[1], T());
        mma_16816(o[2 * cp + 1], pa[ks], b[2], b[3], T());
        if constexpr (std::is_same<T, __nv_bfloat16>::value) {
          mma_16816(o[2 * cp], pl[ks], b[0], b[1], T());
          mma_16816(o[2 * cp + 1], pl[ks], b[2], b[3], T());
        }
      }
    __syncthreads();  // the buffer is refilled two blocks later
  }
  pdl_trigger();
  // row sums across the quad, then the output and the log2-sum-exp
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l[r] += __shfl_xor_sync(kFull, l[r], 1);
    l[r] += __shfl_xor_sync(kFull, l[r], 2);
  }
  const float inv[2] = {l[0] > 0.0f ? 1.0f / l[0] : 0.0f, l[1] > 0.0f ? 1.0f / l[1] : 0.0f};
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = r ? row_g8 : row_g;
    if (row >= p.L) continue;
    float* orow = p.out + ((long long)row * p.Hq + h) * 128;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
      *reinterpret_cast<float2*>(orow + 8 * nt + 2 * qd) = make_float2(o[nt][2 * r] * inv[r], o[nt][2 * r + 1] * inv[r]);
    if (qd == 0) p.lse[(long long)h * p.L + row] = m[r] + __log2f(l[r]);
  }
}

// ---------------------------------------------------------------- pass 2

template <typename T>
__global__ void __launch_bounds__(kThreads) prefill_score(const __grid_constant__ PrefillParams p) {
  extern __shared__ __align__(128) uint8_t smem[];  // K tile | 2 x (Q tile, lse[64])
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, qd = lane & 3;
  const int kb = blockIdx.x;  // the first key blocks see the most query blocks: scheduled first
  const int kvh = blockIdx.y;
  const int k0 = kb * kRows;
  const long long qs = (long long)p.Hq * 128, ks_ = (long long)p.Hkv * 128;
  const int nqb = (p.L + kRows - 1) / kRows;
  uint8_t* Kt = smem;
  float* lse_s = reinterpret_cast<float*>(smem + kTile + 2 * kTile);  // [2][64]
  load_tile(Kt, p.k + (long long)k0 * ks_ + kvh * 128, ks_, min(kRows, p.L - k0), tid);
  // work list: (head, query block) for the gqa heads and the query blocks kb .. nqb - 1
  const int per_head = nqb - kb, total = per_head * p.gqa;
  auto issue = [&](int it) {
    const int h = kvh * p.gqa + it / per_head, qb = kb + it % per_head;
    const int q0 = qb * kRows;
    uint8_t* Qn = smem + kTile + (it & 1) * kTile;
    load_tile(Qn, p.q + (long long)q0 * qs + h * 128, qs, min(kRows, p.L - q0), tid);
    if (tid < kRows) lse_s[(it & 1) * kRows + tid] = q0 + tid < p.L ? p.lse[(long long)h * p.L + q0 + tid] : 0.0f;
  };
  issue(0);
  cp_commit();
  uint32_t ka[8][4];
  float acc[2] = {0.0f, 0.0f};
  const int r0 = warp * 16;
  const int key_g = k0 + r0 + g, key_g8 = key_g + 8;
  for (int it = 0; it < total; ++it) {
    if (it + 1 < total) {
      __syncthreads();  // the buffer of it + 1 was read at it - 1
      issue(it + 1);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    if (it == 0) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) ld_a(ka[ks], Kt, r0, ks, lane);
    }
    const uint8_t* Qt = smem + kTile + (it & 1) * kTile;
    const float* lq = lse_s + (it & 1) * kRows;
    const int q0 = (kb + it % per_head) * kRows;
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) s[i][j] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b[4];
        ld_b_rows(b, Qt, 16 * np, ks, lane);
        mma_16816(s[2 * np], ka[ks], b[0], b[1], T());
        mma_16816(s[2 * np + 1], ka[ks], b[2], b[3], T());
      }
    // P^T[key][query] = 2^(c s - lse[query]) for query >= key (and query < L)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float2 lv = *reinterpret_cast<const float2*>(lq + 8 * nt + 2 * qd);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int query = q0 + 8 * nt + 2 * qd + (j & 1);
        const int key = (j >> 1) ? key_g8 : key_g;
        if (query >= key && query < p.L) acc[j >> 1] += ex2(fmaf(s[nt][j], p.c_log2, -((j & 1) ? lv.y : lv.x)));
      }
    }
  }
  pdl_trigger();
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    acc[r] += __shfl_xor_sync(kFull, acc[r], 1);
    acc[r] += __shfl_xor_sync(kFull, acc[r], 2);
    const int key = r ? key_g8 : key_g;
    if (qd == 0 && key < p.L) p.score[(long long)kvh * p.L + key] = acc[r];
  }
}

// ---------------------------------------------------------------- retention

constexpr int kRetThreads = 1024;

// Exclusive prefix of x over the CTA (position order) and the CTA total.
__device__ __forceinline__ int block_scan(int x, int* s_warp, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(kFull, incl, off);
    if (lane >= off) incl += y;
  }
  __syncthreads();
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int before = 0, sum = 0;
  for (int w = 0; w < kRetThreads / 32; ++w) {
    const int v = s_warp[w];
    if (w < warp) before += v;
    sum += v;
  }
  total = sum;
  return before + incl - x;
}

// One CTA per KV head.  Scores are non-negative fp32, so their bit patterns order like
// their values: a radix select (8 bits at a time, most significant first) finds the
// n_heavy-th largest score T among positions [0, cut) and how many positions equal to T
// are taken (the lowest ones); then one pass in position order writes the kept positions.
__global__ void __launch_bounds__(kRetThreads) retain_kernel(const float* score, int L, int n_heavy, int n_recent,
                                                             int32_t* keep, int32_t* n_keep) {
  pdl_wait();
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need;
  __shared__ int s_warp[kRetThreads / 32];
  const int h = blockIdx.x, tid = threadIdx.x;
  const uint32_t* a = reinterpret_cast<const uint32_t*>(score) + (long long)h * L;
  const int nr = min(max(n_recent, 0), L), cut = L - nr, nh = min(max(n_heavy, 0), cut);
  uint32_t prefix = 0, mask = 0;
  int need = nh;
  if (nh > 0) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kRetThreads) hist[i] = 0;
      __syncthreads();
      for (int j = tid; j < cut; j += kRetThreads) {
        const uint32_t u = __ldcg(a + j);
        if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (tid == 0) {
        int cum = 0;
        for (int d = 255; d >= 0; --d) {
          const int c = int(hist[d]);
          if (cum + c >= need) {
            s_prefix = prefix | (uint32_t(d) << shift);
            s_need = need - cum;
            break;
          }
          cum += c;
        }
      }
      __syncthreads();
      prefix = s_prefix;
      need = s_need;
      mask |= 255u << shift;
      __syncthreads();
    }
  }
  // prefix = T; the first `need` positions equal to T (in position order) are taken
  int eq_before = 0, kept_before = 0;
  for (int base = 0; base < L; base += kRetThreads) {
    const int j = base + tid;
    const uint32_t u = (j < cut && nh > 0) ? __ldcg(a + j) : 0u;
    const int is_eq = (j < cut && nh > 0 && u == prefix) ? 1 : 0;
    int eq_tot;
    const int eqr = eq_before + block_scan(is_eq, s_warp, eq_tot);
    const int kept = (j < L && (j >= cut || (j < cut && nh > 0 && (u > prefix || (is_eq && eqr < need))))) ? 1 : 0;
    int kept_tot;
    const int kpos = kept_before + block_scan(kept, s_warp, kept_tot);
    if (kept) keep[(long long)h * L + kpos] = j;
    eq_before += eq_tot;
    kept_before += kept_tot;
  }
  if (tid == 0) n_keep[h] = kept_before;
  pdl_trigger();
}

// Kept tokens compacted: out[t][h][c] = src[keep[h][t]][h][c] for t < n (one CTA per
// (t, h), 16 threads of 16 bytes).
__global__ void gather_kernel(const uint4* k, const uint4* v, int Hkv, int L, const int32_t* keep, int n,
                              uint4* k_out, uint4* v_out, int32_t* err) {
  pdl_wait();
  const int t = blockIdx.x, h = blockIdx.y, c = threadIdx.x & 15, which = threadIdx.x >> 4;
  int j = keep[(long long)h * L + t];
  if (j < 0 || j >= L) {
    if (threadIdx.x == 0) flag_error(err, KVQ_DEV_ERR_LENGTH);
    j = 0;
  }
  const uint4* src = which ? v : k;
  uint4* dst = which ? v_out : k_out;
  dst[((long long)t * Hkv + h) * 16 + c] = src[((long long)j * Hkv + h) * 16 + c];
  pdl_trigger();
}

}  // namespace pf

// ---------------------------------------------------------------- host side

cudaError_t launch_prefill(const void* q, const void* k, const void* v, int L, int Hq, int Hkv, float sm_scale,
                           int dtype, float* out, float* lse, float* score, cudaStream_t stream) {
  pf::PrefillParams p{};
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.L = L;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.gqa = Hq / Hkv;
  p.c_log2 = sm_scale * 1.4426950408889634f;
  p.out = out;
  p.lse = lse;
  p.score = score;
  const int nb = (L + pf::kRows - 1) / pf::kRows;
  const size_t smem_fwd = 5 * pf::kTile, smem_score = 3 * pf::kTile + 2 * pf::kRows * sizeof(float);
  static int seen[4][64];
  cudaError_t e;
  if (dtype == KVQ_BF16) {
    if ((e = ensure_dynamic_smem(pf::prefill_fwd<__nv_bfloat16>, int(smem_fwd), seen[0])) != cudaSuccess) return e;
    if ((e = ensure_dynamic_smem(pf::prefill_score<__nv_bfloat16>, int(smem_score), seen[1])) != cudaSuccess) return e;
    if ((e = launch_pdl(pf::prefill_fwd<__nv_bfloat16>, dim3(nb, Hq), dim3(pf::kThreads), smem_fwd, stream, p)) !=
        cudaSuccess)
      return e;
    return launch_pdl(pf::prefill_score<__nv_bfloat16>, dim3(nb, Hkv), dim3(pf::kThreads), smem_score, stream, p);
  }
  if ((e = ensure_dynamic_smem(pf::prefill_fwd<__half>, int(smem_fwd), seen[2])) != cudaSuccess) return e;
  if ((e = ensure_dynamic_smem(pf::prefill_score<__half>, int(smem_score), seen[3])) != cudaSuccess) return e;
  if ((e = launch_pdl(pf::prefill_fwd<__half>, dim3(nb, Hq), dim3(pf::kThreads), smem_fwd, stream, p)) != cudaSuccess)
    return e;
  return launch_pdl(pf::prefill_score<__half>, dim3(nb, Hkv), dim3(pf::kThreads), smem_score, stream, p);
}

cudaError_t launch_retain(const float* score, int L, int Hkv, int n_heavy, int n_recent, int32_t* keep,
                          int32_t* n_keep, cudaStream_t stream) {
  return launch_pdl(pf::retain_kernel, dim3(Hkv), dim3(pf::kRetThreads), 0, stream, score, L, n_heavy, n_recent, keep,
                    n_keep);
}

cudaError_t launch_gather(const void* k, const void* v, int Hkv, int L, const int32_t* keep, int n, void* k_out,
                          void* v_out, int32_t* err, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  return launch_pdl(pf::gather_kernel, dim3(n, Hkv), dim3(32), 0, stream, static_cast<const uint4*>(k),
                    static_cast<const uint4*>(v), Hkv, L, keep, n, static_cast<uint4*>(k_out),
                    static_cast<uint4*>(v_out), err);
}

}  // namespace kvq
