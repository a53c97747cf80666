// Decode-attention kernels for fp16 caches with 8 query heads per kv head.
#include "kvq_decode_impl.cuh"

namespace kvq {
KVQ_DECODE_INSTANCE(f16_g8, __half, 8)
}  // namespace kvq
