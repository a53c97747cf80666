// Decode-attention kernels for bf16 caches with 8 query heads per kv head.
#include "kvq_decode_impl.cuh"

namespace kvq {
KVQ_DECODE_INSTANCE(bf16_g8, __nv_bfloat16, 8)
}  // namespace kvq
