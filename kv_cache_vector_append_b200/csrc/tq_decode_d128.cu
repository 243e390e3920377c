// Decode kernels for head_dim 128 (one translation unit per head dimension).
#include "tq_launch.cuh"

namespace tq {
tq_status launch_decode_d128(int kb, int vb, const DecodeParams& p, const DecodePlan& plan,
                            const CUtensorMap& tmap, int64_t steps_upper, cudaStream_t st) {
  return launch_decode_dim<128>(kb, vb, p, plan, tmap, steps_upper, st);
}
}  // namespace tq
