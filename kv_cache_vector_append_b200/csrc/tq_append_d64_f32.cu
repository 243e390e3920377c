// Quantize-append kernels for head_dim 64, f32 input.
#include "tq_append_launch.cuh"

namespace tq {
TQ_DEFINE_APPEND(64, f32, float)
}  // namespace tq
