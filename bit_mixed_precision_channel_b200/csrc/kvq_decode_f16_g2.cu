// Decode-attention kernels for fp16 caches with 2 query heads per kv head.
#include "kvq_decode_impl.cuh"

namespace kvq {
KVQ_DECODE_INSTANCE(f16_g2, __half, 2)
}  // namespace kvq
