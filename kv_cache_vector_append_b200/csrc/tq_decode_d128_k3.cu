// Decode kernels for head_dim 128 and 3-bit K codes (every V width).
#include "tq_launch.cuh"

namespace tq {
TQ_DEFINE_DECODE(128, 3)
}  // namespace tq
