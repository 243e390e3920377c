// Decode kernels for head_dim 256 and 8-bit K codes (every V width).
#include "tq_launch.cuh"

namespace tq {
TQ_DEFINE_DECODE(256, 8)
}  // namespace tq
