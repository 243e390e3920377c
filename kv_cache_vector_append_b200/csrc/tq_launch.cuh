// tq_launch.cuh -- host-side launch helpers shared by the translation units of
// libtq.so (the kernels of each head dimension are compiled separately).
#pragma once

#include <cuda_runtime.h>

#include <algorithm>

#include "tq.h"
#include "tq_append.cuh"
#include "tq_decode.cuh"

namespace tq {

struct DeviceInfo {
  int num_sms = 0;
  int max_smem_optin = 0;
};

struct DecodePlan {
  int wph = 1;        // warps (sub-streams) per KV head
  int nsplit = 1;     // splits per sequence
  int spb = 1;        // blocks per split
  int nstage = 4;     // pipeline depth
  size_t smem = 0;    // dynamic shared memory of the decode kernel
  size_t ws_bytes = 0;
};

inline tq_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

tq_status launch_append_any(int dim, int dtype, const AppendParams& p, const DeviceInfo& di,
                            cudaStream_t st);
tq_status launch_rotate_any(int dim, int dtype, const RotateParams& p, const DeviceInfo& di,
                            cudaStream_t st);
tq_status launch_decode_d64(int kb, int vb, const DecodeParams& p, const MergeParams& m,
                            const DecodePlan& plan, cudaStream_t st);
tq_status launch_decode_d128(int kb, int vb, const DecodeParams& p, const MergeParams& m,
                             const DecodePlan& plan, cudaStream_t st);
tq_status launch_decode_d256(int kb, int vb, const DecodeParams& p, const MergeParams& m,
                             const DecodePlan& plan, cudaStream_t st);

// (K bits, V bits) pairs with a compiled decode kernel.
inline bool decode_bits_supported(int kb, int vb) {
  const int ok[][2] = {{2, 2}, {3, 3}, {4, 4}, {8, 8}, {4, 2}, {3, 2}, {8, 4}, {4, 3}};
  for (auto& c : ok)
    if (c[0] == kb && c[1] == vb) return true;
  return false;
}

template <int D, int KB, int VB, int NH, int NS>
tq_status launch_decode_t(const DecodeParams& p, const MergeParams& m, const DecodePlan& plan,
                          cudaStream_t st) {
  auto kern = decode_kernel<D, KB, VB, NH, NS>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem) !=
      cudaSuccess)
    return TQ_ERR_CUDA;
  dim3 grid(plan.nsplit, p.batch);
  kern<<<grid, p.h_kv * plan.wph * 32, plan.smem, st>>>(p);
  tq_status s = launch_status();
  if (s != TQ_OK) return s;
  merge_kernel<D><<<dim3(p.h_q, p.batch), D, 0, st>>>(m);
  return launch_status();
}

template <int D, int KB, int VB>
tq_status launch_decode_bits(const DecodeParams& p, const MergeParams& m, const DecodePlan& plan,
                             cudaStream_t st) {
  const bool nh2 = p.group > 8;
  if (plan.nstage == 4)
    return nh2 ? launch_decode_t<D, KB, VB, 2, 4>(p, m, plan, st)
               : launch_decode_t<D, KB, VB, 1, 4>(p, m, plan, st);
  return nh2 ? launch_decode_t<D, KB, VB, 2, 2>(p, m, plan, st)
             : launch_decode_t<D, KB, VB, 1, 2>(p, m, plan, st);
}

template <int D>
tq_status launch_decode_dim(int kb, int vb, const DecodeParams& p, const MergeParams& m,
                            const DecodePlan& plan, cudaStream_t st) {
#define TQ_BITS_CASE(KB_, VB_) \
  if (kb == KB_ && vb == VB_) return launch_decode_bits<D, KB_, VB_>(p, m, plan, st);
  TQ_BITS_CASE(2, 2)
  TQ_BITS_CASE(3, 3)
  TQ_BITS_CASE(4, 4)
  TQ_BITS_CASE(8, 8)
  TQ_BITS_CASE(4, 2)
  TQ_BITS_CASE(3, 2)
  TQ_BITS_CASE(8, 4)
  TQ_BITS_CASE(4, 3)
#undef TQ_BITS_CASE
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace tq
