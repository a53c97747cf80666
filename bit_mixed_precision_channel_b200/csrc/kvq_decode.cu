// kvq_decode.cu — host side of decode attention: occupancy of each kernel
// instantiation and the launch (the kernels are in kvq_decode_impl.cuh).
#include "kvq_internal.cuh"

namespace kvq {

cudaError_t decode_occupancy_f16_g1(int kb, int P, int* n);
cudaError_t decode_launch_f16_g1(const DecodeParams& p, cudaStream_t stream);
cudaError_t decode_occupancy_f16_g2(int kb, int P, int* n);
cudaError_t decode_launch_f16_g2(const DecodeParams& p, cudaStream_t stream);
cudaError_t decode_occupancy_f16_g4(int kb, int P, int* n);
cudaError_t decode_launch_f16_g4(const DecodeParams& p, cudaStream_t stream);
cudaError_t decode_occupancy_f16_g8(int kb, int P, int* n);
cudaError_t decode_launch_f16_g8(const DecodeParams& p, cudaStream_t stream);
cudaError_t decode_occupancy_bf16_g1(int kb, int P, int* n);
cudaError_t decode_launch_bf16_g1(const DecodeParams& p, cudaStream_t stream);
cudaError_t decode_occupancy_bf16_g2(int kb, int P, int* n);
cudaError_t decode_launch_bf16_g2(const DecodeParams& p, cudaStream_t stream);
cudaError_t decode_occupancy_bf16_g4(int kb, int P, int* n);
cudaError_t decode_launch_bf16_g4(const DecodeParams& p, cudaStream_t stream);
cudaError_t decode_occupancy_bf16_g8(int kb, int P, int* n);
cudaError_t decode_launch_bf16_g8(const DecodeParams& p, cudaStream_t stream);

static cudaError_t decode_occupancy(int gqa, int dtype, int kb, int P, int* n) {
  const bool bf = dtype == KVQ_BF16;
  switch (gqa) {
    case 1: return bf ? decode_occupancy_bf16_g1(kb, P, n) : decode_occupancy_f16_g1(kb, P, n);
    case 2: return bf ? decode_occupancy_bf16_g2(kb, P, n) : decode_occupancy_f16_g2(kb, P, n);
    case 4: return bf ? decode_occupancy_bf16_g4(kb, P, n) : decode_occupancy_f16_g4(kb, P, n);
    case 8: return bf ? decode_occupancy_bf16_g8(kb, P, n) : decode_occupancy_f16_g8(kb, P, n);
  }
  return cudaErrorInvalidValue;
}

// Resident decode CTAs per SM for a configuration, cached per device and instantiation;
// without a device, the most that 128-thread CTAs can reach (16), so that workspace
// sizes computed there are an upper bound.
int decode_ctas_per_sm(int gqa, int dtype, int kb, int P) {
  static int cache[64][2][4][5][3];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 16;
  }
  const int gi = gqa == 1 ? 0 : gqa == 2 ? 1 : gqa == 4 ? 2 : 3;
  const int ki = kb == 0 ? 0 : kb == 1 ? 1 : kb == 2 ? 2 : kb == 4 ? 3 : 4;
  const int pi = P == 32 ? 0 : P == 64 ? 1 : 2;
  int* slot = &cache[dev][dtype == KVQ_BF16][gi][ki][pi];
  int n = __atomic_load_n(slot, __ATOMIC_ACQUIRE);
  if (n > 0) return n;
  if (decode_occupancy(gqa, dtype, kb, P, &n) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 16;
  }
  __atomic_store_n(slot, n, __ATOMIC_RELEASE);
  return n;
}

cudaError_t launch_decode(const DecodeParams& p, int gqa, int dtype, cudaStream_t stream) {
  if (p.batch <= 0 || p.n_ctas <= 0) return cudaSuccess;
  const bool bf = dtype == KVQ_BF16;
  switch (gqa) {
    case 1: return bf ? decode_launch_bf16_g1(p, stream) : decode_launch_f16_g1(p, stream);
    case 2: return bf ? decode_launch_bf16_g2(p, stream) : decode_launch_f16_g2(p, stream);
    case 4: return bf ? decode_launch_bf16_g4(p, stream) : decode_launch_f16_g4(p, stream);
    case 8: return bf ? decode_launch_bf16_g8(p, stream) : decode_launch_f16_g8(p, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kvq
