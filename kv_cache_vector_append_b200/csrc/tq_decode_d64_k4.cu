// Decode kernels for head_dim 64 and 4-bit K codes (every V width).
#include "tq_launch.cuh"

namespace tq {
TQ_DEFINE_DECODE(64, 4)
}  // namespace tq
