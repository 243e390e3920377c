// Dispatch of quantize-append and the rotation export over (head_dim, dtype);
// the kernels themselves are compiled in tq_append_d<D>_<dtype>.cu.
#include "tq_append_launch.cuh"

namespace tq {

tq_status launch_append_any(int dim, int dtype, const AppendParams& p, const AppendMaps& maps,
                            const DeviceInfo& di, cudaStream_t st) {
#define TQ_CASE(D_, NAME_, T_)                                              \
  if (dim == D_ && dtype == (std::is_same<T_, float>::value ? TQ_F32         \
                             : std::is_same<T_, __half>::value ? TQ_F16       \
                                                               : TQ_BF16))   \
    return launch_append_d##D_##_##NAME_(p, maps, di, st);
  TQ_FOR_EACH_APPEND(TQ_CASE)
#undef TQ_CASE
  return TQ_ERR_UNSUPPORTED;
}

tq_status launch_rotate_any(int dim, int dtype, const RotateParams& p, const DeviceInfo& di,
                            cudaStream_t st) {
#define TQ_CASE(D_, NAME_, T_)                                              \
  if (dim == D_ && dtype == (std::is_same<T_, float>::value ? TQ_F32         \
                             : std::is_same<T_, __half>::value ? TQ_F16       \
                                                               : TQ_BF16))   \
    return launch_rotate_d##D_##_##NAME_(p, di, st);
  TQ_FOR_EACH_APPEND(TQ_CASE)
#undef TQ_CASE
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace tq
