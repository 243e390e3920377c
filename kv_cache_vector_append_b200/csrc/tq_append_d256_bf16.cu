// Quantize-append kernels for head_dim 256, bf16 input.
#include "tq_append_launch.cuh"

namespace tq {
TQ_DEFINE_APPEND(256, bf16, __nv_bfloat16)
}  // namespace tq
