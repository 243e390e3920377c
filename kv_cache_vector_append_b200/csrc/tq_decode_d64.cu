// Decode kernels for head_dim 64 (one translation unit per head dimension).
#include "tq_launch.cuh"

namespace tq {
tq_status launch_decode_d64(int kb, int vb, const DecodeParams& p, const DecodePlan& plan,
                            const CUtensorMap& tmap, int64_t steps_upper, cudaStream_t st) {
  return launch_decode_dim<64>(kb, vb, p, plan, tmap, steps_upper, st);
}
}  // namespace tq
