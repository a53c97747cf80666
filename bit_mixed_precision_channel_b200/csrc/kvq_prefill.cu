// kvq_prefill.cu — prefill attention with cumulative attention scores, token retention
// and the gather of the kept tokens (sm_100a).
//
// MiniKV summary (f-binder), "proposed method": the prompt is processed at prefill, the
// tokens to keep are chosen by their cumulative attention score (heavy hitters) together
// with a recent window, and a two-stage selective flash-attention kernel returns the
// attention output and those scores in linear memory.  Here:
//   pass 1 (prefill_fwd_tc) causal flash attention on the fifth-generation tensor cores
//                          (tcgen05, accumulators in tensor memory), one CTA per (128
//                          query rows, query head): the output rows and each row's
//                          log2-sum-exp;
//   pass 2 (prefill_score_tc) one CTA per (128 key rows, query head), also on tcgen05:
//                          recomputes K Q^T for the query blocks at or after the key
//                          block, turns it into probabilities with the rows' log2-sum-exp
//                          and sums them per key — no L x L matrix is kept; score_heads
//                          adds the query heads of each KV head;
//   retain_kernel          per KV head: the last n_recent positions plus the n_heavy
//                          best-scored others (radix select on the fp32 scores, ties to the
//                          lower position), ascending;
//   gather_kernel          the kept tokens of every KV head, compacted token-major, ready
//                          for the page quantizer.
// Both passes run on tcgen05 (M = N = 128 products, operands in the cache dtype, fp32
// accumulators in tensor memory).  fp16 probabilities carry 11 bits, bf16 ones are split
// into a high and a low bf16 part.
#include <type_traits>

#include "kvq_internal.cuh"
#include "kvq_tc.cuh"

namespace kvq {
namespace pf {

__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

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
  float* part;        // [Hq][L]: cumulative scores per query head (pass 2)
  float* score;       // [Hkv][L]
};

// ---------------------------------------------------------------- pass 1 (tcgen05)

constexpr int kTcRows = 128;                 // query rows per CTA, keys per block
constexpr uint32_t kTcTile = kTcRows * 256;  // one [128][128] tile of the 16-bit dtype

// Byte offset of 16-byte chunk c (8 elements) of row r in a tile built from the tensor
// cores' core matrices: 8 rows x 16 bytes each, chunks 128 bytes apart, row groups 2048
// bytes apart.  The same tile is a K-major operand (rows along M or N, chunks along K:
// LBO = 128, SBO = 2048) and an MN-major one (rows along K, chunks along N: LBO = 2048,
// SBO = 128).
__device__ __forceinline__ uint32_t tco(int r, int c) { return uint32_t((r >> 3) * 2048 + c * 128 + (r & 7) * 16); }

// Rows [0, valid) of a 128-row tile (row i at src + i * stride elements) into shared
// memory with cp.async; rows at or past `valid` are zero-filled.
__device__ __forceinline__ void load_tile_tc(uint8_t* dst, const uint16_t* src, long long stride, int valid, int tid,
                                             int nthreads) {
#pragma unroll 4
  for (int i = tid; i < kTcRows * 16; i += nthreads) {
    const int r = i >> 4, c = i & 15;
    const bool ok = r < valid;
    cp_async16(dst + tco(r, c), src + (ok ? r : 0) * stride + c * 8, ok ? 16u : 0u);
  }
}

constexpr int kTcThreads = 128;  // one thread per query row

// Causal flash attention on the fifth-generation tensor cores: one CTA per (128 query
// rows, query head), thread t owns query row t (tensor-memory lane t).
//   S = Q K^T   M = N = K = 128: Q and K from shared memory (K-major), S in tensor memory;
//   softmax     each thread reads its row of S, masks the diagonal block, keeps a running
//               maximum that is raised only when a block exceeds it by more than 2^8 (O is
//               then rescaled), and writes the probabilities in the cache dtype back over S
//               as the A operand of the next product (bf16: a high and a low part);
//   O += P V    A = P from tensor memory, V from shared memory (MN-major), O in tensor
//               memory.
// Two CTAs share an SM (256 tensor-memory columns and 96 KB of shared memory each), so
// one CTA's softmax runs while the other's products do.  The next K block loads while the
// softmax and PV run, the next V block while the next QK and softmax run.  Every wait is
// bounded; a CTA whose wait gives up writes NaN rows.
template <typename T>
__global__ void __launch_bounds__(kTcThreads, 1) prefill_fwd_tc(const __grid_constant__ PrefillParams p) {
  constexpr bool BF = std::is_same<T, __nv_bfloat16>::value;
  extern __shared__ __align__(128) uint8_t smem[];  // Q, K, V tiles
  __shared__ uint64_t bar_s, bar_o;
  __shared__ uint32_t tmem_base;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int qb = gridDim.x - 1 - blockIdx.x;  // the longest rows first
  const int h = blockIdx.y, kvh = h / p.gqa;
  const int q0 = qb * kTcRows, row = q0 + tid;
  const long long qs = (long long)p.Hq * 128, ks_ = (long long)p.Hkv * 128;
  uint8_t* Qt = smem;
  uint8_t* Kt = smem + kTcTile;
  uint8_t* Vt = smem + 2 * kTcTile;
  if (warp == 0) tc::alloc(&tmem_base, 256);
  if (tid == 0) {
    mbar_init(&bar_s, 1);
    mbar_init(&bar_o, 1);
    fence_mbar_init();
  }
  pdl_wait();
  load_tile_tc(Qt, p.q + (long long)q0 * qs + h * 128, qs, min(kTcRows, p.L - q0), tid, kTcThreads);
  load_tile_tc(Kt, p.k + kvh * 128, ks_, min(kTcRows, p.L), tid, kTcThreads);
  cp_commit();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tS = tmem_base, tO = tmem_base + 128;
  const uint32_t sQ = smem_addr(Qt), sK = smem_addr(Kt), sV = smem_addr(Vt);
  constexpr uint32_t kIdQK = tc::idesc_f16(128, BF, false);
  constexpr uint32_t kIdPV = tc::idesc_f16(128, BF, true);
  float m = -INFINITY, l = 0.0f;
  bool ok = true;

  for (int kb = 0; kb <= qb; ++kb) {
    // the previous PV product is done: its P (over S) and the V buffer are free
    if (kb > 0) {
      ok = mbar_wait_bounded(&bar_o, uint32_t(kb - 1) & 1u) && ok;
      tc::fence_after();
    }
    const int k0 = kb * kTcRows;
    load_tile_tc(Vt, p.v + (long long)k0 * ks_ + kvh * 128, ks_, min(kTcRows, p.L - k0), tid, kTcThreads);
    cp_commit();
    cp_wait<1>();  // Q and this K block landed
    tc::fence_async_smem();
    tc::fence_before();
    __syncthreads();
    if (tid == 0) {
      tc::fence_after();
#pragma unroll
      for (int s = 0; s < 8; ++s)
        tc::mma_ss(tS, tc::smem_desc(sQ + s * 256, 128, 2048), tc::smem_desc(sK + s * 256, 128, 2048), kIdQK,
                   s > 0 ? 1u : 0u);
      tc::commit(&bar_s);
    }
    ok = mbar_wait_bounded(&bar_s, uint32_t(kb) & 1u) && ok;
    tc::fence_after();
    // the K buffer is free: the next key block (an empty group after the last)
    if (kb < qb)
      load_tile_tc(Kt, p.k + (long long)(k0 + kTcRows) * ks_ + kvh * 128, ks_, min(kTcRows, p.L - k0 - kTcRows), tid,
                   kTcThreads);
    cp_commit();

    // this thread's row of S: causal mask and key range (the diagonal block only: every
    // key of an earlier block precedes every row); eight partial maxima of the raw scores
    uint32_t sv[8][16];
#pragma unroll
    for (int i = 0; i < 8; ++i) tc::ld<16>(tc::lane_addr(tS, warp, 16 * i), sv[i]);
    tc::wait_ld();
    float mp[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      mp[i] = -INFINITY;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (kb == qb) {
          const int key = k0 + 16 * i + j;
          if (!(key <= row && key < p.L)) sv[i][j] = 0xff800000u;  // -inf
        }
        mp[i] = fmaxf(mp[i], __uint_as_float(sv[i][j]));
      }
    }
    const float mx =  // the scale is positive: the maximum of the scaled scores
        fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])), fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7]))) *
        p.c_log2;
    // lazy running maximum; O (when it holds earlier blocks) is rescaled with it
    float alpha = 1.0f;
    if (mx > m + 8.0f) {
      alpha = ex2(m - mx);  // m = -inf: 0
      l *= alpha;
      m = mx;
    }
    if (kb > 0 && __any_sync(kFull, alpha != 1.0f)) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint32_t o[16];
        tc::ld<16>(tc::lane_addr(tO, warp, 16 * i), o);
        tc::wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
        tc::st<16>(tc::lane_addr(tO, warp, 16 * i), o);
      }
    }
    // probabilities 2^(s c - m) over S (a masked -inf gives 0): column j holds keys 2j,
    // 2j + 1 (bf16: low parts at 64 + j); m is finite from the first block on
    const float nm = -m;
    float lp[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t ph[16], plo[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int c = 32 * i + 2 * j;  // key offsets c, c + 1
        const float p0 = ex2(__fmaf_rn(__uint_as_float(sv[c >> 4][c & 15]), p.c_log2, nm));
        const float p1 = ex2(__fmaf_rn(__uint_as_float(sv[(c + 1) >> 4][(c + 1) & 15]), p.c_log2, nm));
        lp[i] += p0 + p1;
        ph[j] = pk(p0, p1, T());
        if constexpr (BF) {
          const float2 hv = upk(ph[j], T());
          plo[j] = pk(p0 - hv.x, p1 - hv.y, T());
        }
      }
      tc::st<16>(tc::lane_addr(tS, warp, 16 * i), ph);
      if constexpr (BF) tc::st<16>(tc::lane_addr(tS, warp, 64 + 16 * i), plo);
    }
    l += (lp[0] + lp[1]) + (lp[2] + lp[3]);
    tc::wait_st();
    cp_wait<1>();  // this V block landed (the next K block may still be in flight)
    tc::fence_async_smem();
    tc::fence_before();
    __syncthreads();
    if (tid == 0) {
      tc::fence_after();
#pragma unroll
      for (int s = 0; s < 8; ++s)
        tc::mma(tO, tS + 8 * s, tc::smem_desc(sV + s * 4096, 2048, 128), kIdPV, (kb > 0 || s > 0) ? 1u : 0u);
      if constexpr (BF) {
#pragma unroll
        for (int s = 0; s < 8; ++s) tc::mma(tO, tS + 64 + 8 * s, tc::smem_desc(sV + s * 4096, 2048, 128), kIdPV, 1u);
      }
      tc::commit(&bar_o);
    }
  }
  ok = mbar_wait_bounded(&bar_o, uint32_t(qb) & 1u) && ok;
  tc::fence_after();
  pdl_trigger();
  // the output row and its log2-sum-exp
  const float inv = ok ? (l > 0.0f ? 1.0f / l : 0.0f) : __int_as_float(0x7fc00000);
  float* orow = p.out + ((long long)row * p.Hq + h) * 128;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t o[16];
    tc::ld<16>(tc::lane_addr(tO, warp, 16 * i), o);
    tc::wait_ld();
    if (row < p.L) {
#pragma unroll
      for (int j = 0; j < 16; j += 4)
        *reinterpret_cast<float4*>(orow + 16 * i + j) =
            make_float4(__uint_as_float(o[j]) * inv, __uint_as_float(o[j + 1]) * inv, __uint_as_float(o[j + 2]) * inv,
                        __uint_as_float(o[j + 3]) * inv);
    }
  }
  if (row < p.L) p.lse[(long long)h * p.L + row] = ok ? m + __log2f(l) : __int_as_float(0x7fc00000);
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::dealloc(tmem_base, 256);
}

// ---------------------------------------------------------------- pass 2 (tcgen05)

// Cumulative attention scores on the fifth-generation tensor cores: one CTA per (128 key
// rows, query head), thread t owns key k0 + t (tensor-memory lane t).  For every query
// block at or after the key block:
//   S^T = K Q^T  M = keys, N = queries, K = 128: both tiles from shared memory (K-major),
//               S^T in tensor memory;
//   each thread reads its row of S^T and adds 2^(c s - lse[query]) over the queries that
//   see its key (query >= key, query < L), with lse the row's log2-sum-exp from pass 1.
// The products of the next query block run while the current block is summed (two S^T
// buffers of 128 columns, two query tiles).  A CTA writes its head's sums to part[h];
// score_heads then adds the query heads of each KV head in order, so the scores do not
// depend on scheduling.  Every wait is bounded; a CTA whose wait gives up writes NaN.
template <typename T>
__global__ void __launch_bounds__(kTcThreads, 1) prefill_score_tc(const __grid_constant__ PrefillParams p) {
  constexpr bool BF = std::is_same<T, __nv_bfloat16>::value;
  extern __shared__ __align__(128) uint8_t smem[];  // K tile, 2 query tiles, 3 x lse[128]
  __shared__ uint64_t bar[2];
  __shared__ uint32_t tmem_base;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int kb = blockIdx.x;  // the first key blocks see the most query blocks: scheduled first
  const int h = blockIdx.y, kvh = h / p.gqa;
  const int k0 = kb * kTcRows, key = k0 + tid;
  const long long qs = (long long)p.Hq * 128, ks_ = (long long)p.Hkv * 128;
  const int n = (p.L + kTcRows - 1) / kTcRows - kb;  // query blocks kb .. nqb - 1
  uint8_t* Kt = smem;
  float* lse_s = reinterpret_cast<float*>(smem + 3 * kTcTile);
  if (warp == 0) tc::alloc(&tmem_base, 256);
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  pdl_wait();
  // query block kb + i: its tile into buffer i % 2, its log2-sum-exp into slot i % 3
  auto load_q = [&](int i) {
    const int q0 = (kb + i) * kTcRows;
    load_tile_tc(smem + (1 + (i & 1)) * kTcTile, p.q + (long long)q0 * qs + h * 128, qs, min(kTcRows, p.L - q0), tid,
                 kTcThreads);
    lse_s[(i % 3) * kTcRows + tid] = q0 + tid < p.L ? p.lse[(long long)h * p.L + q0 + tid] : 0.0f;
  };
  load_tile_tc(Kt, p.k + (long long)k0 * ks_ + kvh * 128, ks_, min(kTcRows, p.L - k0), tid, kTcThreads);
  load_q(0);
  cp_commit();
  if (n > 1) load_q(1);
  cp_commit();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t sK = smem_addr(Kt), sQ = smem_addr(smem + kTcTile);
  constexpr uint32_t kId = tc::idesc_f16(128, BF, false);
  auto products = [&](int i) {  // one thread: S^T of query block i into buffer i % 2
    tc::fence_after();
#pragma unroll
    for (int s = 0; s < 8; ++s)
      tc::mma_ss(tmem_base + (i & 1) * 128, tc::smem_desc(sK + s * 256, 128, 2048),
                 tc::smem_desc(sQ + (i & 1) * kTcTile + s * 256, 128, 2048), kId, s > 0 ? 1u : 0u);
    tc::commit(&bar[i & 1]);
  };
  cp_wait<1>();  // the key tile and query block 0 landed
  tc::fence_async_smem();
  tc::fence_before();
  __syncthreads();
  if (tid == 0) products(0);
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  bool ok = true;
  for (int i = 0; i < n; ++i) {
    if (i + 1 < n) {  // the next block's products run while this one is summed
      cp_wait<0>();
      tc::fence_async_smem();
      tc::fence_before();
      __syncthreads();
      if (tid == 0) products(i + 1);
    }
    ok = mbar_wait_bounded(&bar[i & 1], uint32_t(i >> 1) & 1u) && ok;
    tc::fence_after();
    // the products of block i are done: its query buffer takes block i + 2, which loads
    // while this block is summed (its log2-sum-exp slot held block i - 1's, which every
    // thread finished before the barrier that preceded the products of block i + 1)
    if (i + 2 < n) load_q(i + 2);
    cp_commit();
    uint32_t sv[8][16];
#pragma unroll
    for (int j = 0; j < 8; ++j) tc::ld<16>(tc::lane_addr(tmem_base + (i & 1) * 128, warp, 16 * j), sv[j]);
    tc::wait_ld();
    const float* lq = lse_s + (i % 3) * kTcRows;
    const int q0 = (kb + i) * kTcRows;
    if (i == 0 || q0 + kTcRows > p.L) {  // the diagonal block, or the last one: masks
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int query = q0 + 16 * j + c;
          if (query >= key && query < p.L)
            acc[c & 3] += ex2(__fmaf_rn(__uint_as_float(sv[j][c]), p.c_log2, -lq[16 * j + c]));
        }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int c = 0; c < 16; ++c)
          acc[c & 3] += ex2(__fmaf_rn(__uint_as_float(sv[j][c]), p.c_log2, -lq[16 * j + c]));
    }
    // S^T(i) is overwritten by the products of block i + 2, issued after the barrier at
    // the top of the next iteration
  }
  pdl_trigger();
  if (key < p.L)
    p.part[(long long)h * p.L + key] = ok ? (acc[0] + acc[1]) + (acc[2] + acc[3]) : __int_as_float(0x7fc00000);
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::dealloc(tmem_base, 256);
}

// score[kvh][j] = sum over the query heads of kvh of part[h][j], in head order.
__global__ void __launch_bounds__(256) score_heads(const __grid_constant__ PrefillParams p) {
  pdl_wait();
  const int j = blockIdx.x * 256 + threadIdx.x, kvh = blockIdx.y;
  if (j < p.L) {
    float s = 0.0f;
    for (int g = 0; g < p.gqa; ++g) s += p.part[(long long)(kvh * p.gqa + g) * p.L + j];
    p.score[(long long)kvh * p.L + j] = s;
  }
  pdl_trigger();
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
  p.part = lse + size_t(Hq) * L;
  p.score = score;
  const int nb = (L + pf::kTcRows - 1) / pf::kTcRows;
  const size_t smem_fwd = 3 * pf::kTcTile, smem_score = 3 * pf::kTcTile + 3 * pf::kTcRows * sizeof(float);
  static int seen[4][64];
  cudaError_t e;
  if (dtype == KVQ_BF16) {
    if ((e = ensure_dynamic_smem(pf::prefill_fwd_tc<__nv_bfloat16>, int(smem_fwd), seen[0])) != cudaSuccess) return e;
    if ((e = ensure_dynamic_smem(pf::prefill_score_tc<__nv_bfloat16>, int(smem_score), seen[1])) != cudaSuccess)
      return e;
    if ((e = launch_pdl(pf::prefill_fwd_tc<__nv_bfloat16>, dim3(nb, Hq), dim3(pf::kTcThreads), smem_fwd, stream, p)) !=
        cudaSuccess)
      return e;
    if ((e = launch_pdl(pf::prefill_score_tc<__nv_bfloat16>, dim3(nb, Hq), dim3(pf::kTcThreads), smem_score, stream,
                        p)) != cudaSuccess)
      return e;
  } else {
    if ((e = ensure_dynamic_smem(pf::prefill_fwd_tc<__half>, int(smem_fwd), seen[2])) != cudaSuccess) return e;
    if ((e = ensure_dynamic_smem(pf::prefill_score_tc<__half>, int(smem_score), seen[3])) != cudaSuccess) return e;
    if ((e = launch_pdl(pf::prefill_fwd_tc<__half>, dim3(nb, Hq), dim3(pf::kTcThreads), smem_fwd, stream, p)) !=
        cudaSuccess)
      return e;
    if ((e = launch_pdl(pf::prefill_score_tc<__half>, dim3(nb, Hq), dim3(pf::kTcThreads), smem_score, stream, p)) !=
        cudaSuccess)
      return e;
  }
  return launch_pdl(pf::score_heads, dim3((L + 255) / 256, Hkv), dim3(256), 0, stream, p);
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
