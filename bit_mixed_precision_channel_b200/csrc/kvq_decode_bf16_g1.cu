// Decode-attention kernels for bf16 caches with 1 query head per kv head.
#include "kvq_decode_impl.cuh"

namespace kvq {
KVQ_DECODE_INSTANCE(bf16_g1, __nv_bfloat16, 1)
}  // namespace kvq
