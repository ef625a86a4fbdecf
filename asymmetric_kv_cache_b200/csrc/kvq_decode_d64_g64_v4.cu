// Instantiations of the quantized decode kernels for head_dim 64, group
// 64, 4-bit values (2- and 4-bit keys).
#include "kvq_decode_kernels.cuh"

namespace kvq {
KVQ_DECODE_DEFINE(64, 4, 4, 64)
KVQ_DECODE_DEFINE(64, 2, 4, 64)
}  // namespace kvq
