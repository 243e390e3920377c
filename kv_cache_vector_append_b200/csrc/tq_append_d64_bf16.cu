// Quantize-append kernels for head_dim 64, bf16 input.
#include "tq_append_launch.cuh"

namespace tq {
TQ_DEFINE_APPEND(64, bf16, __nv_bfloat16)
}  // namespace tq
