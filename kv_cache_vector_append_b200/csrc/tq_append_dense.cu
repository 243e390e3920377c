// Quantize-append with the dense rotation (tcgen05 tensor cores): host launchers for
// head_dim 64 and 128.
#include "tq_append_dense.cuh"
#include "tq_launch.cuh"

namespace tq {

template <int D>
tq_status launch_append_dense_t(const DenseAppendParams& p0, const DenseAppendMaps& maps,
                                const DeviceInfo& di, cudaStream_t st) {
  DenseAppendParams p = p0;
  const int kb = p.export_mode ? 1 : p.bits[0], vb = p.export_mode ? 1 : p.bits[1];
  p.nst = 2;
  size_t smem = DenseSmem<D>::bytes(kb, vb, 2);
  if ((int)smem > di.max_smem_optin) {
    p.nst = 1;
    smem = DenseSmem<D>::bytes(kb, vb, 1);
    if ((int)smem > di.max_smem_optin) return TQ_ERR_UNSUPPORTED;
  }
  auto kern = append_dense_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return TQ_ERR_CUDA;
  const int64_t ntiles = (p.num_tokens * p.h_kv + kDenseRows - 1) / kDenseRows;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(ntiles, di.num_sms));
  kern<<<grid, kDenseThreads, smem, st>>>(p, maps);
  return launch_status();
}

tq_status launch_append_dense_any(int dim, const DenseAppendParams& p, const DenseAppendMaps& maps,
                                  const DeviceInfo& di, cudaStream_t st) {
  if (dim == 64) return launch_append_dense_t<64>(p, maps, di, st);
  if (dim == 128) return launch_append_dense_t<128>(p, maps, di, st);
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace tq
