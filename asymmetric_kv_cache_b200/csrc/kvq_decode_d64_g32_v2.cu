// Instantiations of the quantized decode kernels for head_dim 64, group
// 32, 2-bit values (2- and 4-bit keys).
#include "kvq_decode_kernels.cuh"

namespace kvq {
KVQ_DECODE_DEFINE(64, 4, 2, 32)
KVQ_DECODE_DEFINE(64, 2, 2, 32)
}  // namespace kvq
