// kvq_tc.cuh — thin inline-PTX wrappers for the fifth-generation tensor cores of
// sm_100a (tcgen05): tensor-memory allocation, loads and stores between registers and
// tensor memory, matrix products with A in tensor memory or shared memory and B in
// shared memory, and completion tracking through an mbarrier.
//
// Operand layouts used by the library (one CTA, M = 128):
//  * A in tensor memory: row m of A is lane m; the 16-bit elements 2j and 2j + 1 of a
//    row sit in column j (low and high half).  One product step reads 16 elements of
//    K, i.e. 8 columns.
//  * Operands in shared memory, no swizzle, built from core matrices of 8 rows x 16
//    bytes (8 elements of the contiguous dimension):
//      - K-major (K contiguous): element (r, k) of an R x K operand at
//        (r / 8) * SBO + (k / 8) * LBO + (r % 8) * 16 + (k % 8) * 2;
//      - MN-major (N contiguous): element (k, n) of a K x N operand at
//        (k / 8) * LBO + (n / 8) * SBO + (k % 8) * 16 + (n % 8) * 2.
//  * D (fp32) in tensor memory: row m is lane m, column n is column n.
// A warp reaches only its own quarter of the lanes: warp w of the CTA accesses lanes
// 32 * (w % 4) .. 32 * (w % 4) + 31.
#pragma once
#include "kvq_internal.cuh"

namespace kvq {
namespace tc {

// Tensor-memory address of column `col` in the lane quarter of warp `w`.
__device__ __forceinline__ uint32_t lane_addr(uint32_t base, int w, int col) {
  return base + (uint32_t(32 * (w & 3)) << 16) + uint32_t(col);
}

// Allocation (one whole warp; the address lands in shared memory).
__device__ __forceinline__ void alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void dealloc(uint32_t base, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols) : "memory");
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// Orders this thread's generic-proxy shared-memory writes before later reads by the
// tensor cores (async proxy).
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 32 lanes x N columns of 32 bits: thread i of the warp holds lane (quarter + i).
template <int N>
__device__ __forceinline__ void ld(uint32_t a, uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void ld<1>(uint32_t a, uint32_t (&r)[1]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r[0]) : "r"(a) : "memory");
}
template <>
__device__ __forceinline__ void ld<2>(uint32_t a, uint32_t (&r)[2]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(a) : "memory");
}
template <>
__device__ __forceinline__ void ld<4>(uint32_t a, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a)
               : "memory");
}
template <>
__device__ __forceinline__ void ld<8>(uint32_t a, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(a)
               : "memory");
}
template <>
__device__ __forceinline__ void ld<16>(uint32_t a, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(a)
      : "memory");
}

template <int N>
__device__ __forceinline__ void st(uint32_t a, const uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void st<8>(uint32_t a, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(a), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
template <>
__device__ __forceinline__ void st<16>(uint32_t a, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(a),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
template <>
__device__ __forceinline__ void st<32>(uint32_t a, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(a),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Shared-memory matrix descriptor: start address, LBO and SBO in bytes (multiples of
// 16), no swizzle, descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return uint64_t((addr >> 4) & 0x3fffu) | (uint64_t((lbo >> 4) & 0x3fffu) << 16) |
         (uint64_t((sbo >> 4) & 0x3fffu) << 32) | (uint64_t(1) << 46);
}

// Instruction descriptor of a kind::f16 product: fp32 accumulate, A and B both fp16
// (bf = false) or both bf16 (bf = true), A K-major, B K-major (b_mn = false) or MN-major
// (b_mn = true), M = 128, N as given (a multiple of 16, 16..256).
__host__ __device__ constexpr uint32_t idesc_f16(int N, bool bf, bool b_mn = true) {
  return (1u << 4) | (uint32_t(bf) << 7) | (uint32_t(bf) << 10) | (uint32_t(b_mn) << 16) | (uint32_t(N >> 3) << 17) |
         (uint32_t(128 >> 4) << 24);
}

// D[tmem d] (+)= A[tmem a] x B[smem desc b]; issued by one thread.
__device__ __forceinline__ void mma(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n\t}\n" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(0u)
      : "memory");
}
// D[tmem d] (+)= A[smem desc a] x B[smem desc b]; issued by one thread.
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(0u)
      : "memory");
}
// The mbarrier receives one arrival when every product this thread issued before has
// completed (and its operands have been read).
__device__ __forceinline__ void commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

}  // namespace tc
}  // namespace kvq
