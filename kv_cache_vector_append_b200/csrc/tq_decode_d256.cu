// Decode kernels for head_dim 256 (one translation unit per head dimension).
#include "tq_launch.cuh"

namespace tq {
tq_status launch_decode_d256(int kb, int vb, const DecodeParams& p, const MergeParams& m,
                             const DecodePlan& plan, cudaStream_t st) {
  return launch_decode_dim<256>(kb, vb, p, m, plan, st);
}
}  // namespace tq
