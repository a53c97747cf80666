// Decode-attention kernels for fp16 caches with 4 query heads per kv head.
#include "kvq_decode_impl.cuh"

namespace kvq {
KVQ_DECODE_INSTANCE(f16_g4, __half, 4)
}  // namespace kvq
