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
  int wph = 1;            // warps (sub-streams) per KV head
  int row_pitch = 0;      // padded shared-memory row pitch (bytes)
  int stage_bytes = 0;    // one pipeline stage: wph blocks
  int ids_cap = 0;        // block ids a CTA preloads into shared memory
  int copy_mode = 0;      // 1: 2-D tensor box per block (padded rows); 0: 1-D bulk copy
  int shared_lut = 0;     // K and V share one lookup table
  size_t smem = 0;        // dynamic shared memory of the decode kernel
  int max_ctas = 0;       // upper bound of the persistent grid
  size_t qfrag_off = 0, qscale_off = 0, prefix_off = 0, part_off = 0;
  size_t ws_bytes = 0;
};

inline tq_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

tq_status launch_append_any(int dim, int dtype, const AppendParams& p, const DeviceInfo& di,
                            cudaStream_t st);
tq_status launch_rotate_any(int dim, int dtype, const RotateParams& p, const DeviceInfo& di,
                            cudaStream_t st);
tq_status launch_decode_d64(int kb, int vb, const DecodeParams& p, const QPrepParams& qp,
                            const MergeParams& m, const DecodePlan& plan,
                            const CUtensorMap& tmap, int64_t steps_upper, cudaStream_t st);
tq_status launch_decode_d128(int kb, int vb, const DecodeParams& p, const QPrepParams& qp,
                             const MergeParams& m, const DecodePlan& plan,
                             const CUtensorMap& tmap, int64_t steps_upper, cudaStream_t st);
tq_status launch_decode_d256(int kb, int vb, const DecodeParams& p, const QPrepParams& qp,
                             const MergeParams& m, const DecodePlan& plan,
                             const CUtensorMap& tmap, int64_t steps_upper, cudaStream_t st);

// (K bits, V bits) pairs with a compiled decode kernel.
inline bool decode_bits_supported(int kb, int vb) {
  const int ok[][2] = {{2, 2}, {3, 3}, {4, 4}, {8, 8}, {4, 2}, {3, 2}, {8, 4}, {4, 3}};
  for (auto& c : ok)
    if (c[0] == kb && c[1] == vb) return true;
  return false;
}

template <int D, int KB, int VB, int NH>
tq_status launch_decode_t(DecodeParams p, QPrepParams qp, MergeParams m, const DecodePlan& plan,
                          const CUtensorMap& tmap, int64_t steps_upper, cudaStream_t st) {
  auto kern = decode_kernel<D, KB, VB, NH>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem) !=
      cudaSuccess)
    return TQ_ERR_CUDA;
  const int threads = p.h_kv * plan.wph * 32;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, plan.smem) !=
      cudaSuccess)
    return TQ_ERR_CUDA;
  per_sm = std::max(1, std::min(per_sm, 2));
  int num_sms = plan.max_ctas / 2;
  // persistent grid, but at least two steps per CTA so that tiny batches do not pay
  // one prologue per step
  const int64_t ctas = std::max<int64_t>(
      1, std::min<int64_t>(std::min<int64_t>((int64_t)num_sms * per_sm, plan.max_ctas),
                           (steps_upper + 1) / 2));
  m.nctas = (int32_t)ctas;
  const int qrows = p.batch * p.h_q;
  qprep_kernel<D, KB><<<(qrows + 7) / 8, 256, 0, st>>>(qp, qrows);
  tq_status s = launch_status();
  if (s != TQ_OK) return s;
  kern<<<(unsigned)ctas, threads, plan.smem, st>>>(p, tmap);
  s = launch_status();
  if (s != TQ_OK) return s;
  merge_kernel<D><<<dim3(p.h_q, p.batch), 256, 0, st>>>(m);
  return launch_status();
}

template <int D, int KB, int VB>
tq_status launch_decode_bits(const DecodeParams& p, const QPrepParams& qp, const MergeParams& m,
                             const DecodePlan& plan, const CUtensorMap& tmap,
                             int64_t steps_upper, cudaStream_t st) {
  return p.group > 8 ? launch_decode_t<D, KB, VB, 2>(p, qp, m, plan, tmap, steps_upper, st)
                     : launch_decode_t<D, KB, VB, 1>(p, qp, m, plan, tmap, steps_upper, st);
}

template <int D>
tq_status launch_decode_dim(int kb, int vb, const DecodeParams& p, const QPrepParams& qp,
                            const MergeParams& m, const DecodePlan& plan,
                            const CUtensorMap& tmap, int64_t steps_upper, cudaStream_t st) {
#define TQ_BITS_CASE(KB_, VB_) \
  if (kb == KB_ && vb == VB_)  \
    return launch_decode_bits<D, KB_, VB_>(p, qp, m, plan, tmap, steps_upper, st);
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

// Bytes of the replicated lookup table(s) of the decode kernel.
inline size_t decode_lut_bytes(int kb, int vb, bool shared) {
  auto one = [](int b) { return (size_t)(b <= 4 ? (1 << (2 * b)) : (1 << b)) * 32 * 4; };
  return shared ? one(kb) : one(kb) + one(vb);
}

}  // namespace tq
