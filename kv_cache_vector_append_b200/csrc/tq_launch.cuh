// tq_launch.cuh -- host-side launch helpers shared by the translation units of
// libtq.so (the kernels of each head dimension are compiled separately).
#pragma once

#include <cuda_runtime.h>

#include <algorithm>

#include "tq.h"
#include "tq_append.cuh"
#include "tq_append_dense.cuh"
#include "tq_decode.cuh"

namespace tq {

struct DeviceInfo {
  int num_sms = 0;
  int max_smem_optin = 0;
  uint32_t dyn_smem_base = 0;   // shared-window address where dynamic shared memory starts
                                // (kernels without static shared memory)
};

struct DecodePlan {
  int maxw = 16;          // warps per CTA the kernel is compiled for (16 or 8)
  uint32_t lut_win = 0;   // shared-memory layout (see DecodeParams)
  int lut_off = 0, stage_lo_off = 0, stage_hi_off = 0, n_low = 0, misc_off = 0;
  int wph = 1;            // warps (sub-streams) per KV head
  int nst = 4;            // stages in the ring
  int row_pitch = 0;      // shared-memory row pitch (bytes)
  int stage_bytes = 0;    // one pipeline stage: wph blocks
  int ids_cap = 0;        // block ids a CTA preloads into shared memory
  int copy_mode = 0;      // 1: 2-D tensor box per block (padded rows); 0: 1-D bulk copy
  int lut_bytes = 0;      // lookup tables at the start of shared memory
  size_t smem = 0;        // dynamic shared memory of the decode kernel
  int max_ctas = 0;       // upper bound of the persistent grid (one CTA per SM)
  size_t part_off = 0, counters_off = 0;
  size_t ws_bytes = 0;
};

inline tq_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

tq_status launch_append_any(int dim, int dtype, const AppendParams& p, const AppendMaps& maps,
                            const DeviceInfo& di, cudaStream_t st);
tq_status launch_rotate_any(int dim, int dtype, const RotateParams& p, const DeviceInfo& di,
                            cudaStream_t st);
tq_status launch_append_dense_any(int dim, const DenseAppendParams& p, const DenseAppendMaps& maps,
                                  const DeviceInfo& di, cudaStream_t st);
// Code widths with a compiled decode kernel: K and V independently in {2, 3, 4, 8}.
inline bool decode_bits_supported(int kb, int vb) {
  auto ok = [](int b) { return b == 2 || b == 3 || b == 4 || b == 8; };
  return ok(kb) && ok(vb);
}

template <int D, int KB, int VB, int NH, int MAXW>
tq_status launch_decode_t(const DecodeParams& p, const DecodePlan& plan, const CUtensorMap& tmap,
                          int64_t steps_upper, cudaStream_t st) {
  auto kern = decode_kernel<D, KB, VB, NH, MAXW, 0>;
  if (p.qjl) {
    if constexpr (D >= 128 && KB <= 4) kern = decode_kernel<D, KB, VB, NH, MAXW, 2>;
    else return TQ_ERR_UNSUPPORTED;
  } else if (p.hot_k != nullptr || p.rot_hi != nullptr) {
    kern = decode_kernel<D, KB, VB, NH, MAXW, 1>;
  }
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem) !=
      cudaSuccess)
    return TQ_ERR_CUDA;
  const int threads = p.h_kv * plan.wph * 32;
  // persistent grid of one CTA per SM, but at least two steps per CTA so that tiny
  // batches do not pay one prologue per step
  const int64_t ctas =
      std::max<int64_t>(1, std::min<int64_t>(plan.max_ctas, (steps_upper + 1) / 2));
  // cooperative: the CTAs of a sequence wait for one another before merging it, so all
  // of them must be resident at once
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3((unsigned)threads);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, p, tmap) != cudaSuccess) return TQ_ERR_CUDA;
  return launch_status();
}

// Warps per CTA the decode kernel is compiled for: 16 (<= 128 registers a thread) when
// the per-warp state fits, else 8.
inline int decode_maxw(int dim, int group) { return dim <= 128 && group <= 8 ? 16 : 8; }

template <int D, int KB, int VB>
tq_status launch_decode_bits(const DecodeParams& p, const DecodePlan& plan,
                             const CUtensorMap& tmap, int64_t steps_upper, cudaStream_t st) {
  if (p.group > 8) return launch_decode_t<D, KB, VB, 2, 8>(p, plan, tmap, steps_upper, st);
  if constexpr (D <= 128) return launch_decode_t<D, KB, VB, 1, 16>(p, plan, tmap, steps_upper, st);
  else return launch_decode_t<D, KB, VB, 1, 8>(p, plan, tmap, steps_upper, st);
}

// All V widths for one (head_dim, K width); instantiated in tq_decode_d<D>_k<KB>.cu so
// that the kernels compile in parallel.
template <int D, int KB>
tq_status launch_decode_kbits(int vb, const DecodeParams& p, const DecodePlan& plan,
                              const CUtensorMap& tmap, int64_t steps_upper, cudaStream_t st) {
  switch (vb) {
    case 2: return launch_decode_bits<D, KB, 2>(p, plan, tmap, steps_upper, st);
    case 3: return launch_decode_bits<D, KB, 3>(p, plan, tmap, steps_upper, st);
    case 4: return launch_decode_bits<D, KB, 4>(p, plan, tmap, steps_upper, st);
    case 8: return launch_decode_bits<D, KB, 8>(p, plan, tmap, steps_upper, st);
    default: return TQ_ERR_UNSUPPORTED;
  }
}

#define TQ_FOR_EACH_DECODE(X) \
  X(64, 2) X(64, 3) X(64, 4) X(64, 8) \
  X(128, 2) X(128, 3) X(128, 4) X(128, 8) \
  X(256, 2) X(256, 3) X(256, 4) X(256, 8)
#define TQ_DECLARE_DECODE(D_, KB_)                                                          \
  tq_status launch_decode_d##D_##_k##KB_(int vb, const DecodeParams& p, const DecodePlan& plan, \
                                         const CUtensorMap& tmap, int64_t steps_upper,       \
                                         cudaStream_t st);
#define TQ_DEFINE_DECODE(D_, KB_)                                                           \
  tq_status launch_decode_d##D_##_k##KB_(int vb, const DecodeParams& p, const DecodePlan& plan, \
                                         const CUtensorMap& tmap, int64_t steps_upper,       \
                                         cudaStream_t st) {                                  \
    return launch_decode_kbits<D_, KB_>(vb, p, plan, tmap, steps_upper, st);                 \
  }
TQ_FOR_EACH_DECODE(TQ_DECLARE_DECODE)

// Decode launch for any supported (head_dim, K width, V width).
inline tq_status launch_decode_any(int dim, int kb, int vb, const DecodeParams& p,
                                   const DecodePlan& plan, const CUtensorMap& tmap,
                                   int64_t steps_upper, cudaStream_t st) {
#define TQ_DECODE_CASE(D_, KB_) \
  if (dim == D_ && kb == KB_) return launch_decode_d##D_##_k##KB_(vb, p, plan, tmap, steps_upper, st);
  TQ_FOR_EACH_DECODE(TQ_DECODE_CASE)
#undef TQ_DECODE_CASE
  return TQ_ERR_UNSUPPORTED;
}

// Bytes of the lookup tables of the decode kernel (one 256-byte row per entry).
inline size_t decode_lut_bytes(int kb, int vb) {
  // 2-bit V codes are looked up four at a time (256 entries) where they are read
  // interleaved; the table is sized for that whatever the head dimension
  return (size_t)std::max(lut_entries(kb), vb == 2 ? 256 : lut_entries(vb)) * kLutRow;
}

}  // namespace tq
