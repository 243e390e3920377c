// tq_append_launch.cuh -- host launchers of the append and rotation-export
// kernels, instantiated once per (head_dim, input dtype) translation unit.
#pragma once

#include "tq_launch.cuh"

namespace tq {

// FIXB > 0: the fast path's instantiation for K and V codes of FIXB bits (the redo
// stays generic; both give the same bytes).
template <int D, typename Tin, bool QJL, int FIXB = 0>
tq_status launch_append_q(const AppendParams& p, const AppendMaps& maps, const DeviceInfo& di,
                          cudaStream_t st) {
  const size_t smem = AppendSmem<D, Tin>::bytes(p.bits[0], p.bits[1]);
  if ((int)smem > di.max_smem_optin) return TQ_ERR_UNSUPPORTED;
  auto kern = append_kernel<D, Tin, false, QJL, FIXB>;
  auto kern_safe = append_kernel<D, Tin, true, QJL>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(kern_safe, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess)
    return TQ_ERR_CUDA;
  using G = AppendGeom<D>;
  const int64_t tiles = (p.num_tokens * p.h_kv + G::ROWS - 1) / G::ROWS;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kAppendWarps * 32, smem) !=
      cudaSuccess)
    per_sm = 1;
  per_sm = std::max(per_sm, 1);
  const int64_t max_ctas = (int64_t)di.num_sms * per_sm;
  const int64_t want = (tiles + kAppendWarps - 1) / kAppendWarps;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, max_ctas));
  // the fast path, then the redo that runs only when a row left the fast path's range
  kern<<<grid, kAppendWarps * 32, smem, st>>>(p, maps);
  kern_safe<<<grid, kAppendWarps * 32, smem, st>>>(p, maps);
  return launch_status();
}

// The plain append, or (p.kcent set) the one that also stores the keys' QJL sketch
// (built for head_dim 128 and 256).
template <int D, typename Tin>
tq_status launch_append_t(const AppendParams& p, const AppendMaps& maps, const DeviceInfo& di,
                          cudaStream_t st) {
  if (p.kcent == nullptr) {
    if (p.bits[0] == 4 && p.bits[1] == 4) return launch_append_q<D, Tin, false, 4>(p, maps, di, st);
    return launch_append_q<D, Tin, false>(p, maps, di, st);
  }
  if constexpr (D >= 128) return launch_append_q<D, Tin, true>(p, maps, di, st);
  return TQ_ERR_UNSUPPORTED;
}

template <int D, typename Tin>
tq_status launch_rotate_t(const RotateParams& p, const DeviceInfo& di, cudaStream_t st) {
  using G = AppendGeom<D>;
  const size_t smem = 4 * D + 1024 + kAppendWarps * AppendSmem<D, Tin>::KIND;
  auto kern = rotate_unit_kernel<D, Tin>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return TQ_ERR_CUDA;
  const int64_t tiles = (p.rows + G::ROWS - 1) / G::ROWS;
  const int64_t want = (tiles + kAppendWarps - 1) / kAppendWarps;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)di.num_sms * 4));
  kern<<<grid, kAppendWarps * 32, smem, st>>>(p);
  return launch_status();
}

#define TQ_DECLARE_APPEND(D_, NAME_, T_)                                                  \
  tq_status launch_append_d##D_##_##NAME_(const AppendParams& p, const AppendMaps& maps, \
                                          const DeviceInfo& di, cudaStream_t st);        \
  tq_status launch_rotate_d##D_##_##NAME_(const RotateParams& p, const DeviceInfo& di,   \
                                          cudaStream_t st);
#define TQ_DEFINE_APPEND(D_, NAME_, T_)                                                   \
  tq_status launch_append_d##D_##_##NAME_(const AppendParams& p, const AppendMaps& maps, \
                                          const DeviceInfo& di, cudaStream_t st) {       \
    return launch_append_t<D_, T_>(p, maps, di, st);                                    \
  }                                                                                      \
  tq_status launch_rotate_d##D_##_##NAME_(const RotateParams& p, const DeviceInfo& di,   \
                                          cudaStream_t st) {                             \
    return launch_rotate_t<D_, T_>(p, di, st);                                          \
  }

#define TQ_FOR_EACH_APPEND(X) \
  X(64, bf16, __nv_bfloat16)  \
  X(64, f16, __half)          \
  X(64, f32, float)           \
  X(128, bf16, __nv_bfloat16) \
  X(128, f16, __half)         \
  X(128, f32, float)          \
  X(256, bf16, __nv_bfloat16) \
  X(256, f16, __half)         \
  X(256, f32, float)

TQ_FOR_EACH_APPEND(TQ_DECLARE_APPEND)

}  // namespace tq
