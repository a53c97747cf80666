// Decode-attention kernels for fp16 caches with 1 query head per kv head.
#include "kvq_decode_impl.cuh"

namespace kvq {
KVQ_DECODE_INSTANCE(f16_g1, __half, 1)
}  // namespace kvq
