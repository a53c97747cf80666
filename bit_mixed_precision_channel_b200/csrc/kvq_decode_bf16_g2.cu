// Decode-attention kernels for bf16 caches with 2 query heads per kv head.
#include "kvq_decode_impl.cuh"

namespace kvq {
KVQ_DECODE_INSTANCE(bf16_g2, __nv_bfloat16, 2)
}  // namespace kvq
