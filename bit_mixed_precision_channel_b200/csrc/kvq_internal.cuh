// kvq_internal.cuh — shared device/host helpers of the kvq CUDA library (sm_100a).
//
// Record layout, launch helpers and thin inline-PTX wrappers used by the quantize
// and decode kernels.  Nothing here is exported; the C ABI lives in include/kvq.h.
#pragma once
#include <utility>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

// Weights of the decode kernel's work line, in units of one 32-token page group (a page
// stage of 128 tokens weighs 4).  Measured on B200 (per-CTA traces regressed on the
// items each CTA held): a 16-token residual piece, which one warp processes while the
// stage waits for it, costs about as much time as three page groups; the merge at the
// end of a (sequence, KV head) is given extra weight where no item starts.
constexpr int kDecodePieceWeight = 3;
constexpr int kDecodeMergeWeight = 6;

constexpr int kHeadDim = 128;
constexpr int kKeyGroup = 32;
constexpr unsigned kFull = 0xffffffffu;

// Byte offsets of one (page, kv head) record.  Section order and sizes follow the
// page-record description in kvq.h: plane A codes, plane B codes, value codes, plane-A
// scale and zero, plane-B scale, value scale and zero, boost indices; the stride rounds
// the payload up to 128 bytes so records stay aligned for 16-byte vector access and
// for bulk copies.
struct Layout {
  uint32_t k_codes, kb_codes, v_codes, k_scale, k_zero, kb_scale, v_scale, v_zero, boost_idx;
  uint32_t payload, record;
};

inline Layout make_layout(int P, int D, int k, int G) {
  Layout L;
  uint32_t off = 0;
  L.k_codes = off;   off += uint32_t(P) * uint32_t(D / 16) * 4u;
  L.kb_codes = off;  off += uint32_t(P) * uint32_t(k / 16) * 4u;
  L.v_codes = off;   off += uint32_t(D) * uint32_t(P / 16) * 4u;
  L.k_scale = off;   off += uint32_t(P / G) * uint32_t(D) * 2u;
  L.k_zero = off;    off += uint32_t(P / G) * uint32_t(D) * 2u;
  L.kb_scale = off;  off += uint32_t(P / G) * uint32_t(k) * 2u;
  L.v_scale = off;   off += uint32_t(P) * 2u;
  L.v_zero = off;    off += uint32_t(P) * 2u;
  L.boost_idx = off; off += uint32_t(k);
  L.payload = off;
  L.record = (off + 127u) / 128u * 128u;
  return L;
}

// Storage order of the packed rows (see the page-record description in kvq.h).
// Key channel c = 16s + 8r + 2q + f  <->  plane-A code position 32q + 4s + 2r + f.
__host__ __device__ __forceinline__ int key_pos(int c) {
  return 32 * ((c >> 1) & 3) + 4 * (c >> 4) + 2 * ((c >> 3) & 1) + (c & 1);
}
// ... and k_scale / k_zero position 32*(s>>1) + 8q + 4*(s&1) + 2r + f.
__host__ __device__ __forceinline__ int key_meta_pos(int c) {
  const int s = c >> 4;
  return 32 * (s >> 1) + 8 * ((c >> 1) & 3) + 4 * (s & 1) + 2 * ((c >> 3) & 1) + (c & 1);
}
// Boosted row j = 16s + 8r + 2q + f  <->  position 4*KB*q + 4s + 2r + f.
__host__ __device__ __forceinline__ int boost_pos(int j, int KB) {
  return 4 * KB * ((j >> 1) & 3) + 4 * (j >> 4) + 2 * ((j >> 3) & 1) + (j & 1);
}
// Value scale / zero position of token t = 32g + 8u + w: 32g + 4w + u.
__host__ __device__ __forceinline__ int value_meta_pos(int t) {
  return (t & ~31) + 4 * (t & 7) + ((t >> 3) & 3);
}
// Bit of element e = 8a + 2b + f inside a code word: 8b + 4f + 2a.
__host__ __device__ __forceinline__ int elem_bit(int e) {
  return 8 * ((e >> 1) & 3) + 4 * (e & 1) + 2 * (e >> 3);
}

__device__ __forceinline__ void flag_error(int32_t* err, int bits) {
  if (err) atomicOr(err, bits);
}

// ------------------------------------------------------------------ 16-bit helpers

template <typename T> struct Pair;
template <> struct Pair<__half> { using type = __half2; };
template <> struct Pair<__nv_bfloat16> { using type = __nv_bfloat162; };

__device__ __forceinline__ float bits_to_float(uint16_t b, __half) { return __half2float(__ushort_as_half(b)); }
__device__ __forceinline__ float bits_to_float(uint16_t b, __nv_bfloat16) {
  return __uint_as_float(uint32_t(b) << 16);
}
// Rounds a float toward +infinity to the 16-bit type; returns the bits.
__device__ __forceinline__ uint16_t round_up_bits(float x, __half) { return __half_as_ushort(__float2half_ru(x)); }
__device__ __forceinline__ uint16_t round_up_bits(float x, __nv_bfloat16) {
  return __bfloat16_as_ushort(__float2bfloat16_ru(x));
}
// Exact conversion of a representable float to the 16-bit type.
__device__ __forceinline__ uint16_t exact_bits(float x, __half) { return __half_as_ushort(__float2half_rn(x)); }
__device__ __forceinline__ uint16_t exact_bits(float x, __nv_bfloat16) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// ------------------------------------------------------------------ shared memory access

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint32_t lds32(const void* p) { return *reinterpret_cast<const uint32_t*>(p); }
__device__ __forceinline__ uint2 lds64(const void* p) { return *reinterpret_cast<const uint2*>(p); }
__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }

// ------------------------------------------------------------------ mbarrier + bulk copy

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}
// try_wait that may suspend the thread for up to `ns` nanoseconds while the phase is
// incomplete (fewer spin iterations competing with the warps that compute).
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}
// Waits for the phase of `parity` to complete; gives up after ~2^32 SM cycles
// (about two seconds) and returns false so the caller can flag an error and leave.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait_suspend(bar, parity, 100000u)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_suspend(bar, parity, 100000u)) {
    if (clock64() - t0 > (1ll << 32)) return false;
  }
  return true;
}
// One contiguous global -> shared copy through the bulk-copy engine, completing on `bar`.
// Both addresses 16-byte aligned, bytes a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}
// L2 policy for data read once per launch: evicted first.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 16-byte asynchronous copy global -> shared; src_bytes < 16 zero-fills the rest.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
// The mbarrier receives one arrival once all of this thread's prior cp.async copies
// have landed (its pending count is raised first, so the phase waits for it).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}
// ------------------------------------------------------------------ warp-level matrix ops

// D += A(16x16, row) * B(16x8, col), fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                          __half) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                          __nv_bfloat16) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}

// 2^x (hardware approximation, relative error ~2^-22; -inf -> 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Four fp16 pairs from one masked pass of a code word.  After x = (w >> 2a) & 0x33333333
// every nibble of x holds one 2-bit code in its low bits, which read as an FP4 (e2m1)
// number is exactly 0.5 * code (0, 0.5, 1, 1.5).  The hardware conversion turns each
// byte of x into an fp16 pair (low nibble -> low half): byte b gives elements
// (8a + 2b, 8a + 2b + 1) of the word.  Products with the other operand stay exact;
// the factor 0.5 is undone after the contraction.
constexpr float kCodeScale = 2.0f;  // value of a code / value delivered to the tensor cores
__device__ __forceinline__ void e2m1_pairs(uint32_t x, uint32_t& p0, uint32_t& p1, uint32_t& p2, uint32_t& p3) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(p0), "=r"(p1), "=r"(p2), "=r"(p3)
      : "r"(x));
}
// The fp16 pair of byte 0 of x (x already masked).
__device__ __forceinline__ uint32_t e2m1_pair_lo(uint32_t x) {
  uint32_t d;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t}"
      : "=r"(d)
      : "r"(x));
  return d;
}
__device__ __forceinline__ uint32_t code_pass(uint32_t w, int a) { return (w >> (2 * a)) & 0x33333333u; }

__device__ __forceinline__ uint32_t bf2_as_u32(__nv_bfloat162 h) { return *reinterpret_cast<uint32_t*>(&h); }
// A register of two cache-dtype values as the dtype's pair type, and back.
__device__ __forceinline__ __half2 u32_as_pair(uint32_t x, __half) { return u32_as_h2(x); }
__device__ __forceinline__ __nv_bfloat162 u32_as_pair(uint32_t x, __nv_bfloat16) {
  return *reinterpret_cast<__nv_bfloat162*>(&x);
}
__device__ __forceinline__ uint32_t pair_as_u32(__half2 h) { return h2_as_u32(h); }
__device__ __forceinline__ uint32_t pair_as_u32(__nv_bfloat162 h) { return bf2_as_u32(h); }

// ------------------------------------------------------------------ dependent launches

// Every kernel of the library is launched with programmatic stream serialization: it
// may be scheduled while the kernel before it in the stream is still finishing, and it
// waits for that kernel's completion (griddepcontrol.wait) before it reads anything.
// A kernel signals with pdl_trigger() when the next one may be scheduled.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ------------------------------------------------------------------ launch parameters

enum : int { kModeSelect = 1, kModeKeys = 2, kModeValues = 4 };

// Page quantization (a1..a3) over n items; in flush mode item = sequence b and only
// sequences whose residual window is full are quantized.
struct QuantParams {
  const uint16_t* k_src;
  const uint16_t* v_src;
  long long k_page_stride, k_tok_stride, k_head_stride;  // elements
  long long v_page_stride, v_tok_stride, v_head_stride;
  const int32_t* dst_pages;  // page id per item, or new_page[b] in flush mode
  uint8_t* pool;
  long long pool_pages;
  int Hkv, P, k;
  Layout L;
  int32_t* err;
  int mode;
  int flush;
  const int32_t* res_len;
  const int32_t* num_pages;
  int max_pages;
  const float* qw;     // query-aware ranking weights [Hkv][128], or null (magnitude ranking)
  const int32_t* kh;   // boosted channels per kv head [Hkv] (each <= k), or null (k for all)
  // append-and-flush mode (a4 + a5 in one launch): the new token, the writable window,
  // lengths and page table, and one arrival counter per sequence
  int append;
  const uint16_t* k_new;
  const uint16_t* v_new;
  uint16_t* res_k;
  uint16_t* res_v;
  int32_t* res_len_w;
  int32_t* num_pages_w;
  int32_t* page_table;
  int32_t* counters;
};

// Decode attention (a6 + a7).
struct DecodeParams {
  const uint8_t* pool;
  long long pool_pages;
  int Hkv, P, k, KB;  // KB = k / 16
  Layout L;
  const uint16_t* q;
  int batch, Hq;
  const int32_t* page_table;
  int max_pages;
  const int32_t* num_pages;
  const uint16_t* res_k;
  const uint16_t* res_v;
  const int32_t* res_len;
  float c_log2;  // sm_scale * log2(e)
  float* out;
  float* part;    // [n_ctas + batch * Hkv][GQA][128 + 4]: unnormalised output, max, sum
  uint32_t* cnt;  // [batch * Hkv] arrival counters
  int n_ctas;     // grid size: SMs x resident CTAs per SM
  int n_sms;      // SMs of the device
  int32_t* err;
  // dense mode: tokens per sequence; pool then holds raw pages [pool_pages][Hkv][2][P][128]
  // (K rows, V rows) of the cache dtype, and num_pages / res_len / res_k / res_v are unused
  const int32_t* seq_len;
};

cudaError_t launch_quantize(const QuantParams& p, int n_items, int dtype, cudaStream_t stream);
cudaError_t launch_append(const void* k_new, const void* v_new, void* res_k, void* res_v, int32_t* res_len,
                          int batch, int Hkv, int P, int32_t* err, cudaStream_t stream);
cudaError_t launch_flush_commit(int32_t* res_len, const int32_t* new_page, int32_t* page_table, int max_pages,
                                int32_t* num_pages, long long pool_pages, int batch, int P, cudaStream_t stream);
cudaError_t launch_decode(const DecodeParams& p, int gqa, int dtype, cudaStream_t stream);
cudaError_t launch_prefill(const void* q, const void* k, const void* v, int L, int Hq, int Hkv, float sm_scale,
                           int dtype, float* out, float* lse, float* score, cudaStream_t stream);
cudaError_t launch_retain(const float* score, int L, int Hkv, int n_heavy, int n_recent, int32_t* keep,
                          int32_t* n_keep, cudaStream_t stream);
cudaError_t launch_gather(const void* k, const void* v, int Hkv, int L, const int32_t* keep, int n, void* k_out,
                          void* v_out, int32_t* err, cudaStream_t stream);
int decode_ctas_per_sm(int gqa, int dtype, int kb, int P);

// Raises a kernel's dynamic shared-memory limit once per device and size, so that
// later calls (and calls made while a stream is being captured into a graph) issue
// no attribute call.  `seen` holds the largest size already set, per device.
template <typename Kernel>
inline cudaError_t ensure_dynamic_smem(Kernel kernel, int bytes, int (&seen)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (bytes <= __atomic_load_n(&seen[dev], __ATOMIC_ACQUIRE)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) {
    int cur = __atomic_load_n(&seen[dev], __ATOMIC_ACQUIRE);
    while (cur < bytes && !__atomic_compare_exchange_n(&seen[dev], &cur, bytes, false, __ATOMIC_ACQ_REL,
                                                        __ATOMIC_ACQUIRE)) {
    }
  }
  return e;
}
size_t decode_main_bytes(int P, int GQA, uint32_t rec_bytes);
kvq_status decode_check_args(const kvq_config* cfg, const void* pool, int64_t pool_pages, const void* q,
                             int32_t batch, const int32_t* page_table, int32_t max_pages, const int32_t* num_pages,
                             const void* res_k, const void* res_v, const int32_t* res_len, const float* out);

}  // namespace kvq
