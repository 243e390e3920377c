// tq_api.cu -- the extern "C" boundary of libtq.so (declared in include/tq.h):
// argument validation, kernel dispatch, per-device workspace and error word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "tq.h"
#include "tq_launch.cuh"

namespace tq {

__device__ unsigned int g_tq_error_word;

// Flag and counter of quantize-append's redo (see append_kernel): zero between calls.
__device__ unsigned int g_tq_append_redo[2];

// Scratch of tq_paged_decode_noalloc: a fixed device array that every device which
// loads the library holds until the process exits.  Host code never dereferences
// this name (on the host it is only a stand-in); its device address is looked up
// per device with cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_tq_noalloc_scratch[TQ_NOALLOC_SCRATCH_BYTES];

__device__ unsigned int g_tq_dyn_base;

// Records where dynamic shared memory starts in the shared window of a kernel that
// has no static shared memory (the decode kernel's layout is planned against it).
__global__ void dyn_smem_base_probe() {
  extern __shared__ __align__(16) uint8_t smem[];
  g_tq_dyn_base = (unsigned int)__cvta_generic_to_shared(smem);
}

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  // device address of g_tq_error_word; published (release) last by the one-time set-up,
  // so a non-null value means `info` is complete
  std::atomic<unsigned int*> err{nullptr};
  unsigned int* redo = nullptr;   // device address of g_tq_append_redo
  void* user_ws = nullptr;
  size_t user_ws_bytes = 0;
  void* lib_ws = nullptr;
  size_t lib_ws_bytes = 0;
  uint8_t* noalloc_scratch = nullptr;   // device address of g_tq_noalloc_scratch
  size_t counter_bytes = 0;             // largest merge-counter area a decode call used
  DeviceInfo info;
  // one-shot test hook of the next decode launch (tq_debug_inject_merge_stall)
  int32_t inject_withhold = -1;
  uint32_t inject_wait_ms = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

// The current device's state, set up on first use: the error word's address, the SM
// count, the shared-memory limit and where dynamic shared memory starts.  The set-up
// runs once per device under g_mu; other threads see the state only once it is whole.
tq_status device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TQ_ERR_CUDA;
  DeviceState& s = g_dev[dev];
  if (s.err.load(std::memory_order_acquire) == nullptr) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (s.err.load(std::memory_order_relaxed) == nullptr) {
      void* p = nullptr;
      void* r = nullptr;
      if (cudaGetSymbolAddress(&p, g_tq_error_word) != cudaSuccess ||
          cudaGetSymbolAddress(&r, g_tq_append_redo) != cudaSuccess)
        return TQ_ERR_CUDA;
      s.redo = (unsigned int*)r;
      DeviceInfo info;
      if (cudaDeviceGetAttribute(&info.num_sms, cudaDevAttrMultiProcessorCount, dev) !=
          cudaSuccess)
        return TQ_ERR_CUDA;
      if (cudaDeviceGetAttribute(&info.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                                 dev) != cudaSuccess)
        return TQ_ERR_CUDA;
      dyn_smem_base_probe<<<1, 1, 16>>>();
      unsigned int base = 0;
      if (cudaGetLastError() != cudaSuccess ||
          cudaMemcpyFromSymbol(&base, g_tq_dyn_base, sizeof(base)) != cudaSuccess)
        return TQ_ERR_CUDA;
      info.dyn_smem_base = base;
      s.info = info;
      s.err.store((unsigned int*)p, std::memory_order_release);
    }
  }
  *out = &s;
  return TQ_OK;
}

int dtype_size(int32_t dt) {
  switch (dt) {
    case TQ_U8: return 1;
    case TQ_I32: return 4;
    case TQ_I64: return 8;
    case TQ_F32: return 4;
    case TQ_BF16: return 2;
    case TQ_F16: return 2;
    default: return 0;
  }
}

bool is_float_dtype(int32_t dt) { return dt == TQ_F32 || dt == TQ_BF16 || dt == TQ_F16; }

int region_bytes(int dim, int bits) { return (dim * bits + 7) / 8 + 4; }

bool valid_tensor(const tq_tensor& t, int ndim) {
  if (t.ndim != ndim || t.data == nullptr || dtype_size(t.dtype) == 0) return false;
  for (int i = 0; i < ndim; ++i)
    if (t.shape[i] < 0) return false;
  if ((uintptr_t)t.data % (uintptr_t)dtype_size(t.dtype) != 0) return false;
  return true;
}

bool valid_codebook(const tq_codebook& c, int dim) {
  return c.dim == dim && c.bits >= 1 && c.bits <= 8 && c.centroids != nullptr &&
         c.boundaries != nullptr && (uintptr_t)c.centroids % 4 == 0 &&
         (uintptr_t)c.boundaries % 4 == 0;
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

bool valid_rotation(const tq_rotation* r, int dim) {
  return r != nullptr && r->dim == dim && r->hi != nullptr && r->lo != nullptr &&
         (uintptr_t)r->hi % 16 == 0 && (uintptr_t)r->lo % 16 == 0;
}

// Heads per tensor box of the dense append (a tile is 128 pairs: box_h heads x
// 128 / box_h tokens), or 0 when h_kv neither divides 128 nor is a multiple of it.
int dense_box_heads(int h_kv) {
  if (h_kv <= kDenseRows && kDenseRows % h_kv == 0) return h_kv;
  if (h_kv % kDenseRows == 0) return kDenseRows;
  return 0;
}

// A bf16 [T, H_kv, D] input the dense append reads by tensor copies.
bool dense_input_ok(const tq_tensor& t) {
  return t.dtype == TQ_BF16 && (uintptr_t)t.data % 16 == 0 && t.stride[0] % 8 == 0 &&
         t.stride[1] % 8 == 0;
}

int align_mode_of(const void* data, int esize, std::initializer_list<int64_t> strides) {
  auto ok = [&](int a) {
    if ((uintptr_t)data % a) return false;
    for (int64_t s : strides)
      if ((s * esize) % a) return false;
    return true;
  };
  if (ok(16)) return 16;
  if (ok(4)) return 4;
  return 0;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

int pow2_floor(int x) {
  int r = 1;
  while (2 * r <= x) r *= 2;
  return r;
}

// Geometry of the decode kernel for one call (see tq_decode.cuh).
tq_status plan_decode(int batch, int h_q, int h_kv, int dim, int kb, int vb, int slot_stride,
                      int max_blocks, bool allow_tensor_copy, const DeviceInfo& di,
                      DecodePlan* plan, bool qjl = false) {
  plan->maxw = decode_maxw(dim, h_q / h_kv);
  if (h_kv < 1 || h_kv > plan->maxw) return TQ_ERR_UNSUPPORTED;
  // A block is staged by one TMA copy.  When a row is a multiple of 16 bytes and the
  // padded row fits a tensor box (at most 256 u64 columns), the copy is a 2-D box of
  // 16 rows x pitch/8 u64 whose columns past the row end are zero-filled, giving rows
  // padded to a pitch of 20 (mod 32) words; otherwise it is a 1-D bulk copy of the
  // block with unpadded rows.
  const int row_bytes = h_kv * slot_stride;
  int words = row_bytes / 4;
  words += ((20 - words % 32) + 32) % 32;
  plan->copy_mode = allow_tensor_copy && row_bytes % 16 == 0 && 4 * words / 8 <= 256;
  plan->row_pitch = plan->copy_mode ? 4 * words : row_bytes;
  plan->lut_bytes = (int)decode_lut_bytes(kb, vb);
  plan->max_ctas = di.num_sms;
  const int wph_max = pow2_floor(plan->maxw / h_kv);
  // The dynamic shared memory spans shared-window addresses [base, base + budget).  The
  // tables go to a multiple of 65536 inside it; the stages fill the space below and
  // above them; the misc area (barriers, q', prefix sums, block ids, merge partials)
  // goes at the bottom or at the top, whichever leaves more stages.
  const int64_t base = di.dyn_smem_base;
  const int64_t budget = (int64_t)di.max_smem_optin;
  const int64_t lut = plan->lut_bytes;
  bool found = false;
  for (int wph = wph_max; wph >= 1 && !found; wph /= 2) {
    const int64_t stage = (int64_t)wph * kBlockSize * plan->row_pitch;
    const int64_t steps_upper = (int64_t)batch * ((max_blocks + wph - 1) / wph);
    const int64_t per_cta = (steps_upper + di.num_sms - 1) / di.num_sms + 1;
    const int ids_cap = (int)std::min<int64_t>(per_cta * wph, 4096);
    const int min_st = wph == 1 ? 2 : 4;
    int best_nst = 0;
    int64_t best_end = 0;
    DecodePlan best;
    for (int64_t L = 65536; L + lut <= base + budget; L += 65536) {
      if (L < base) continue;
      const int64_t low = L - base, high = base + budget - (L + lut);
      for (int nst = kMaxStages; nst >= min_st; --nst) {
        const int64_t misc = 16 * nst + 2LL * h_q * dim + 4LL * h_q + 4LL * (batch + 1) +
                             4LL * ids_cap + 4 * 36 + (int64_t)plan->maxw * (dim + 2) * 4 +
                             4LL * dim + 4LL * batch + 32 +
                             (qjl ? ((int64_t)h_q * qjl_qz_stride(dim) + 15) / 16 * 16 : 0);
        for (int at_top = 0; at_top < 2; ++at_top) {
          const int64_t below = at_top ? low : low - misc;   // room for stages below
          if (below < 0) continue;
          const int nl = (int)std::min<int64_t>(nst, below / stage);
          const int nh = nst - nl;
          const int64_t hi_off = (L - base) + lut;
          const int64_t misc_off = at_top ? (hi_off + nh * stage + 15) / 16 * 16 : 0;
          const int64_t end = at_top ? misc_off + misc : (nh > 0 ? hi_off + nh * stage : hi_off);
          if (end > budget) continue;
          if (nst > best_nst || (nst == best_nst && end < best_end)) {
            best_nst = nst;
            best_end = end;
            best.lut_win = (uint32_t)L;
            best.lut_off = (int)(L - base);
            best.stage_lo_off = (int)(L - base - nl * stage);
            best.stage_hi_off = (int)hi_off;
            best.n_low = nl;
            best.misc_off = (int)misc_off;
          }
        }
        if (best_nst == nst) break;        // the deepest ring this L allows
      }
    }
    if (best_nst > 0) {
      plan->wph = wph;
      plan->nst = best_nst;
      plan->stage_bytes = (int)stage;
      plan->ids_cap = ids_cap;
      plan->smem = (size_t)best_end;
      plan->lut_win = best.lut_win;
      plan->lut_off = best.lut_off;
      plan->stage_lo_off = best.stage_lo_off;
      plan->stage_hi_off = best.stage_hi_off;
      plan->n_low = best.n_low;
      plan->misc_off = best.misc_off;
      found = true;
    }
  }
  if (!found) return TQ_ERR_UNSUPPORTED;
  // workspace: merge counters (at the start, so that they can be cleared without
  // knowing a call's geometry: per sequence, covering CTAs that published and heads
  // finished), then the partial records (sized for the widest step)
  plan->counters_off = 0;
  plan->part_off = align256((size_t)batch * 2 * sizeof(unsigned int));
  plan->ws_bytes = plan->part_off + (size_t)(plan->max_ctas + batch) * wph_max * h_q * (dim + 4) *
                                        sizeof(float);
  return TQ_OK;
}

// cuTensorMapEncodeTiled, looked up once through the runtime (no link against libcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// Tensor map of the page pool seen as (num_blocks * 16) rows of row_bytes / 8 u64
// columns, read in boxes of 16 rows x pitch / 8 columns (columns past the row end are
// out of bounds and zero-filled).  Returns false when the driver rejects the map.
bool encode_page_map(CUtensorMap* map, const void* pages, int64_t num_blocks, int row_bytes,
                     int pitch) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (fn == nullptr || num_blocks * kBlockSize > 0xffffffffll) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)(row_bytes / 8), (cuuint64_t)(num_blocks * kBlockSize)};
  const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  const cuuint32_t box[2] = {(cuuint32_t)(pitch / 8), (cuuint32_t)kBlockSize};
  const cuuint32_t estride[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<void*>(pages), dims, strides, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map of a (tokens, h_kv, D) 16-bit K or V input seen as (D, h_kv, tokens)
// elements, read in boxes of 64 elements x `box_h` heads x `box_t` tokens with the
// 128-byte swizzle.  Returns false when the driver rejects the map.
bool encode_input_map(CUtensorMap* map, const void* data, int64_t T, int h_kv, int D,
                      int64_t tok_stride, int64_t head_stride, int box_h, int box_t) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (fn == nullptr || T > 0x7fffffffll) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)h_kv, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)(head_stride * 2), (cuuint64_t)(tok_stride * 2)};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_h, (cuuint32_t)box_t};
  const cuuint32_t estride[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(data), dims, strides, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DecodeCall {
  int B = 0, h_q = 0, h_kv = 0, D = 0, kbits = 0, vbits = 0, kb = 0, max_blocks = 0;
  bool qjl = false;
  int64_t stride = 0;
  DeviceState* ds = nullptr;
  DecodePlan plan;
};

// Validation and geometry of one decode call (shared by the decode entry points).
tq_status decode_prepare(const tq_tensor& out, const tq_tensor& q, const tq_tensor& pages,
                         const tq_tensor& block_table, const tq_tensor& seq_lens,
                         const tq_codebooks* cb, float scale, DecodeCall* call,
                         bool qjl = false) {
  if (cb == nullptr || !std::isfinite(scale)) return TQ_ERR_INVALID_ARG;
  if (!valid_tensor(q, 3) || !is_float_dtype(q.dtype) || q.stride[2] != 1) return TQ_ERR_INVALID_ARG;
  if (!valid_tensor(out, 3) || !is_float_dtype(out.dtype) || out.stride[2] != 1 ||
      (out.dtype != TQ_F32 && out.dtype != q.dtype))
    return TQ_ERR_INVALID_ARG;
  if (!valid_tensor(pages, 4) || pages.dtype != TQ_U8) return TQ_ERR_INVALID_ARG;
  if (!valid_tensor(block_table, 2) || block_table.dtype != TQ_I32 || block_table.stride[1] != 1)
    return TQ_ERR_INVALID_ARG;
  if (!valid_tensor(seq_lens, 1) || seq_lens.dtype != TQ_I32 || seq_lens.stride[0] != 1)
    return TQ_ERR_INVALID_ARG;
  // (sequence, query head) pairs are counted in 32 bits
  if (q.shape[0] * q.shape[1] >= (int64_t)1 << 31) return TQ_ERR_UNSUPPORTED;
  const int B = (int)q.shape[0], h_q = (int)q.shape[1], D = (int)q.shape[2];
  const int h_kv = (int)pages.shape[2];
  for (int i = 0; i < 3; ++i)
    if (out.shape[i] != q.shape[i]) return TQ_ERR_INVALID_ARG;
  if (block_table.shape[0] != B || seq_lens.shape[0] != B) return TQ_ERR_INVALID_ARG;
  if (h_kv < 1 || h_q % h_kv) return TQ_ERR_INVALID_ARG;
  if (!valid_codebook(cb->k, D) || !valid_codebook(cb->v, D)) return TQ_ERR_INVALID_ARG;
  const int kbits = cb->k.bits, vbits = cb->v.bits;
  const int kb = region_bytes(D, kbits) + (qjl ? D / 8 + 4 : 0), vb = region_bytes(D, vbits);
  const int64_t stride = pages.shape[3];
  if (stride < kb + vb || stride % 8) return TQ_ERR_INVALID_ARG;
  // contiguous page tensor: whole blocks are staged with 16-byte copies
  if (pages.stride[3] != 1 || pages.stride[2] != stride || pages.stride[1] != h_kv * stride ||
      pages.stride[0] != pages.shape[1] * h_kv * stride || (uintptr_t)pages.data % 16)
    return TQ_ERR_INVALID_ARG;
  if (pages.shape[1] != kBlockSize) return TQ_ERR_UNSUPPORTED;
  if (D != 64 && D != 128 && D != 256) return TQ_ERR_UNSUPPORTED;
  if (h_q / h_kv > 16 || h_kv > decode_maxw(D, h_q / h_kv)) return TQ_ERR_UNSUPPORTED;
  if (!decode_bits_supported(kbits, vbits)) return TQ_ERR_UNSUPPORTED;
  if (qjl && (D == 64 || kbits > 4)) return TQ_ERR_UNSUPPORTED;
  call->qjl = qjl;
  call->B = B;
  if (B == 0) return TQ_OK;
  DeviceState* ds = nullptr;
  tq_status s = device_state(&ds);
  if (s != TQ_OK) return s;
  const int max_blocks = (int)block_table.shape[1];
  DecodePlan plan;
  s = plan_decode(B, h_q, h_kv, D, kbits, vbits, (int)stride, std::max(max_blocks, 1), true,
                  ds->info, &plan, qjl);
  if (s != TQ_OK) return s;
  if ((h_kv * stride) % 8) return TQ_ERR_INVALID_ARG;
  call->h_q = h_q;
  call->h_kv = h_kv;
  call->D = D;
  call->kbits = kbits;
  call->vbits = vbits;
  call->kb = kb;
  call->stride = stride;
  call->max_blocks = max_blocks;
  call->ds = ds;
  call->plan = plan;
  return TQ_OK;
}

// Optional uncompressed hot window of a decode call.
struct HotWindow {
  const tq_tensor* k = nullptr;
  const tq_tensor* v = nullptr;
  const tq_tensor* lens = nullptr;
};

// Validation of a hot window against a prepared call: k and v [B, W, H_kv, D] of one
// float dtype with equal strides and a contiguous last dim, lens i32 [B] contiguous.
tq_status hot_validate(const DecodeCall& call, const tq_tensor& q, const HotWindow& hw) {
  const tq_tensor &k = *hw.k, &v = *hw.v, &n = *hw.lens;
  if (!valid_tensor(k, 4) || !valid_tensor(v, 4) || !is_float_dtype(k.dtype) ||
      k.dtype != v.dtype || k.stride[3] != 1)
    return TQ_ERR_INVALID_ARG;
  for (int i = 0; i < 4; ++i)
    if (k.shape[i] != v.shape[i] || k.stride[i] != v.stride[i]) return TQ_ERR_INVALID_ARG;
  if (k.shape[0] != q.shape[0] || k.shape[3] != q.shape[2] || k.shape[1] > 0x7fffffff)
    return TQ_ERR_INVALID_ARG;
  if (call.B > 0 && k.shape[2] != call.h_kv) return TQ_ERR_INVALID_ARG;
  if (!valid_tensor(n, 1) || n.dtype != TQ_I32 || n.stride[0] != 1 || n.shape[0] != q.shape[0])
    return TQ_ERR_INVALID_ARG;
  return TQ_OK;
}

// Launch the decode kernels of a prepared call on workspace `ws` (plan.ws_bytes bytes).
tq_status decode_run(const DecodeCall& call, const tq_tensor& out, const tq_tensor& q,
                     const tq_tensor& pages, const tq_tensor& block_table,
                     const tq_tensor& seq_lens, const tq_codebooks* cb, uint64_t sign_seed,
                     float scale, uint8_t* ws, void* stream, const HotWindow& hw = HotWindow(),
                     const tq_rotation* rot = nullptr, uint64_t qjl_seed = 0) {
  const int B = call.B, h_q = call.h_q, h_kv = call.h_kv, D = call.D;
  const int kbits = call.kbits, vbits = call.vbits, kb = call.kb;
  const int64_t stride = call.stride;
  const int max_blocks = call.max_blocks;
  DeviceState* ds = call.ds;
  DecodePlan plan = call.plan;
  CUtensorMap tmap;
  std::memset(&tmap, 0, sizeof(tmap));
  if (plan.copy_mode &&
      !encode_page_map(&tmap, pages.data, pages.shape[0], h_kv * (int)stride, plan.row_pitch)) {
    // the 1-D bulk layout never needs more shared memory or workspace than the 2-D one
    const tq_status s = plan_decode(B, h_q, h_kv, D, kbits, vbits, (int)stride,
                                    std::max(max_blocks, 1), false, ds->info, &plan, call.qjl);
    if (s != TQ_OK) return s;
  }
  DecodeParams p{};
  p.pages = (const uint8_t*)pages.data;
  p.num_blocks = (int32_t)pages.shape[0];
  p.h_kv = h_kv;
  p.slot_stride = (int32_t)stride;
  p.row_pitch = plan.row_pitch;
  p.blk_stride = pages.stride[0];
  p.block_table = (const int32_t*)block_table.data;
  p.bt_stride = block_table.stride[0];
  p.max_blocks = max_blocks;
  p.seq_lens = (const int32_t*)seq_lens.data;
  p.batch = B;
  p.q = q.data;
  p.q_bstride = q.stride[0];
  p.q_hstride = q.stride[1];
  p.q_dtype = q.dtype;
  p.out = out.data;
  p.o_bstride = out.stride[0];
  p.o_hstride = out.stride[1];
  p.out_dtype = out.dtype;
  p.h_q = h_q;
  p.group = h_q / h_kv;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.sign_seed = sign_seed;
  p.kc = cb->k.centroids;
  p.vc = cb->v.centroids;
  p.k_region = kb;
  p.wph = plan.wph;
  p.nst = plan.nst;
  p.stage_bytes = plan.stage_bytes;
  p.ids_cap = plan.ids_cap;
  p.copy_mode = plan.copy_mode;
  p.lut_bytes = plan.lut_bytes;
  p.lut_win = plan.lut_win;
  p.lut_off = plan.lut_off;
  p.stage_lo_off = plan.stage_lo_off;
  p.stage_hi_off = plan.stage_hi_off;
  p.n_low = plan.n_low;
  p.misc_off = plan.misc_off;
  p.smem_end = (int32_t)plan.smem;
  p.part = (float*)(ws + plan.part_off);
  p.counters = (unsigned int*)(ws + plan.counters_off);
  p.wait_ms = kWaitMs;
  p.withhold_cta = -1;
  p.qjl = call.qjl ? 1 : 0;
  p.qjl_seed = qjl_seed;
  p.rot_hi = rot ? rot->hi : nullptr;
  p.rot_lo = rot ? rot->lo : nullptr;
  p.hot_k = nullptr;
  p.hot_v = nullptr;
  p.hot_lens = nullptr;
  if (hw.k != nullptr) {
    p.hot_k = hw.k->data;
    p.hot_v = hw.v->data;
    p.hot_bstride = hw.k->stride[0];
    p.hot_tstride = hw.k->stride[1];
    p.hot_hstride = hw.k->stride[2];
    p.hot_dtype = hw.k->dtype;
    p.hot_cap = (int32_t)hw.k->shape[1];
    p.hot_lens = (const int32_t*)hw.lens->data;
  }
  {
    std::lock_guard<std::mutex> lock(g_mu);
    ds->counter_bytes = std::max(ds->counter_bytes, plan.part_off);
    if (ds->inject_wait_ms > 0) {
      p.wait_ms = ds->inject_wait_ms;
      p.withhold_cta = ds->inject_withhold;
      ds->inject_wait_ms = 0;
      ds->inject_withhold = -1;
    }
  }
  p.err = ds->err.load(std::memory_order_relaxed);

  const int64_t steps_upper = (int64_t)B * ((max_blocks + plan.wph - 1) / plan.wph);
  cudaStream_t st = as_stream(stream);
  return launch_decode_any(D, kbits, vbits, p, plan, tmap, steps_upper, st);
}

// The workspace of a decode call: the caller's (tq_set_workspace) or the library's own,
// grown on demand.
tq_status decode_workspace(const DecodeCall& call, uint8_t** ws) {
  DeviceState* ds = call.ds;
  const DecodePlan& plan = call.plan;
  std::lock_guard<std::mutex> lock(g_mu);
  if (ds->user_ws != nullptr) {
    if (ds->user_ws_bytes < plan.ws_bytes) return TQ_ERR_WORKSPACE;
    *ws = (uint8_t*)ds->user_ws;
    return TQ_OK;
  }
  if (ds->lib_ws_bytes < plan.ws_bytes) {
    if (ds->lib_ws) cudaFree(ds->lib_ws);
    ds->lib_ws = nullptr;
    ds->lib_ws_bytes = 0;
    size_t want = std::max<size_t>(plan.ws_bytes, 1 << 20);
    if (cudaMalloc(&ds->lib_ws, want) != cudaSuccess) return TQ_ERR_WORKSPACE;
    if (cudaMemset(ds->lib_ws, 0, want) != cudaSuccess) return TQ_ERR_CUDA;
    ds->lib_ws_bytes = want;
  }
  *ws = (uint8_t*)ds->lib_ws;
  return TQ_OK;
}

}  // namespace
}  // namespace tq

using namespace tq;

extern "C" {

const char* tq_version(void) { return "0.1.0"; }

const char* tq_status_string(tq_status s) {
  switch (s) {
    case TQ_OK: return "ok";
    case TQ_ERR_INVALID_ARG: return "invalid argument";
    case TQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case TQ_ERR_CUDA: return "CUDA runtime error";
    case TQ_ERR_DEVICE: return "device-side error reported";
    case TQ_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

tq_status tq_slot_bytes(int32_t dim, int32_t k_bits, int32_t v_bits, int32_t* out) {
  if (out == nullptr || dim < 1 || k_bits < 1 || k_bits > 8 || v_bits < 1 || v_bits > 8)
    return TQ_ERR_INVALID_ARG;
  *out = region_bytes(dim, k_bits) + region_bytes(dim, v_bits);
  return TQ_OK;
}

tq_status append_impl(tq_tensor pages, tq_tensor slot_mapping, tq_tensor k, tq_tensor v,
                      const tq_codebooks* cb, uint64_t sign_seed, int32_t k_bits, int32_t v_bits,
                      void* stream, bool qjl, uint64_t qjl_seed);

tq_status tq_quantize_append(tq_tensor pages, tq_tensor slot_mapping, tq_tensor k, tq_tensor v,
                             const tq_codebooks* cb, uint64_t sign_seed, int32_t k_bits,
                             int32_t v_bits, void* stream) {
  return append_impl(pages, slot_mapping, k, v, cb, sign_seed, k_bits, v_bits, stream, false, 0);
}

tq_status tq_quantize_append_qjl(tq_tensor pages, tq_tensor slot_mapping, tq_tensor k,
                                 tq_tensor v, const tq_codebooks* cb, uint64_t sign_seed,
                                 uint64_t qjl_seed, int32_t k_bits, int32_t v_bits, void* stream) {
  return append_impl(pages, slot_mapping, k, v, cb, sign_seed, k_bits, v_bits, stream, true,
                     qjl_seed);
}

tq_status tq_slot_bytes_qjl(int32_t dim, int32_t k_bits, int32_t v_bits, int32_t* out) {
  if (out == nullptr || dim < 8 || dim % 8 || k_bits < 1 || k_bits > 8 || v_bits < 1 ||
      v_bits > 8)
    return TQ_ERR_INVALID_ARG;
  *out = region_bytes(dim, k_bits) + dim / 8 + 4 + region_bytes(dim, v_bits);
  return TQ_OK;
}

tq_status append_impl(tq_tensor pages, tq_tensor slot_mapping, tq_tensor k, tq_tensor v,
                      const tq_codebooks* cb, uint64_t sign_seed, int32_t k_bits, int32_t v_bits,
                      void* stream, bool qjl, uint64_t qjl_seed) {
  if (cb == nullptr) return TQ_ERR_INVALID_ARG;
  if (!valid_tensor(pages, 4) || pages.dtype != TQ_U8 || pages.stride[3] != 1)
    return TQ_ERR_INVALID_ARG;
  if (!valid_tensor(slot_mapping, 1) || slot_mapping.dtype != TQ_I64) return TQ_ERR_INVALID_ARG;
  if (!valid_tensor(k, 3) || !valid_tensor(v, 3) || !is_float_dtype(k.dtype) ||
      k.dtype != v.dtype || k.stride[2] != 1 || v.stride[2] != 1)
    return TQ_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (k.shape[i] != v.shape[i]) return TQ_ERR_INVALID_ARG;
  const int64_t T = k.shape[0];
  const int h_kv = (int)k.shape[1];
  const int D = (int)k.shape[2];
  if (slot_mapping.shape[0] != T || pages.shape[2] != h_kv) return TQ_ERR_INVALID_ARG;
  if (k_bits < 1 || k_bits > 8 || v_bits < 1 || v_bits > 8) return TQ_ERR_INVALID_ARG;
  if (!valid_codebook(cb->k, D) || !valid_codebook(cb->v, D) || cb->k.bits != k_bits ||
      cb->v.bits != v_bits)
    return TQ_ERR_INVALID_ARG;
  if (D != 64 && D != 128 && D != 256) return TQ_ERR_UNSUPPORTED;
  if (qjl && D == 64) return TQ_ERR_UNSUPPORTED;
  const int kb = region_bytes(D, k_bits) + (qjl ? D / 8 + 4 : 0), vb = region_bytes(D, v_bits);
  if (pages.shape[3] < kb + vb || pages.shape[3] % 8 != 0) return TQ_ERR_INVALID_ARG;
  if (pages.stride[0] % 4 || pages.stride[1] % 4 || pages.stride[2] % 4 ||
      (uintptr_t)pages.data % 4)
    return TQ_ERR_INVALID_ARG;
  if (T == 0 || h_kv == 0) return TQ_OK;
  if (T * h_kv >= ((int64_t)1 << 31) - 64) return TQ_ERR_UNSUPPORTED;   // 32-bit row indices
  DeviceState* ds = nullptr;
  tq_status s = device_state(&ds);
  if (s != TQ_OK) return s;

  AppendParams p{};
  p.pages = (uint8_t*)pages.data;
  p.num_slots = pages.shape[0] * pages.shape[1];
  p.block_size = (int32_t)pages.shape[1];
  p.bs_shift = -1;
  for (int sh = 0; sh < 31; ++sh)
    if ((int64_t)1 << sh == pages.shape[1]) p.bs_shift = sh;
  p.h_kv = h_kv;
  p.blk_stride = pages.stride[0];
  p.row_stride = pages.stride[1];
  p.head_stride = pages.stride[2];
  p.slot_mapping = (const int64_t*)slot_mapping.data;
  p.slot_map_stride = slot_mapping.stride[0];
  p.num_tokens = T;
  p.src[0] = k.data;
  p.src[1] = v.data;
  p.tok_stride[0] = k.stride[0];
  p.tok_stride[1] = v.stride[0];
  p.head_stride_in[0] = k.stride[1];
  p.head_stride_in[1] = v.stride[1];
  p.boundaries[0] = cb->k.boundaries;
  p.boundaries[1] = cb->v.boundaries;
  p.bits[0] = k_bits;
  p.bits[1] = v_bits;
  p.region_off[0] = 0;
  p.region_off[1] = kb;
  p.sign_seed = sign_seed;
  p.kcent = qjl ? cb->k.centroids : nullptr;
  p.qjl_seed = qjl_seed;
  p.err = ds->err.load(std::memory_order_relaxed);
  p.redo = ds->redo;
  const int es = dtype_size(k.dtype);
  p.align_mode = std::min(align_mode_of(k.data, es, {k.stride[0], k.stride[1]}),
                          align_mode_of(v.data, es, {v.stride[0], v.stride[1]}));
  if (p.align_mode == 16 &&
      (align_mode_of(k.data, es, {k.stride[0], k.stride[1]}) != 16 ||
       align_mode_of(v.data, es, {v.stride[0], v.stride[1]}) != 16))
    p.align_mode = 4;
  if (k.dtype == TQ_F32 && p.align_mode == 0) return TQ_ERR_INVALID_ARG;

  // Tiles of `rows` consecutive (token, head) pairs are whole runs of one token's heads
  // when h_kv divides rows or rows divides h_kv.
  const int rows = 2048 / D;
  p.run_heads = (h_kv <= rows && rows % h_kv == 0) ? h_kv : (h_kv % rows == 0 ? rows : 0);
  const int slot = kb + vb;
  p.bulk_out = p.run_heads > 0 && pages.shape[3] == slot && pages.stride[2] == slot &&
               (uintptr_t)pages.data % 16 == 0 && pages.stride[0] % 16 == 0 &&
               pages.stride[1] % 16 == 0 && ((int64_t)p.run_heads * slot) % 16 == 0;
  // a padded slot stride: slots stored one by one, the 16-byte body by a bulk copy
  p.slot_body = 0;
  if (!p.bulk_out && slot >= 16 && (uintptr_t)pages.data % 16 == 0 &&
      pages.stride[0] % 16 == 0 && pages.stride[1] % 16 == 0 && pages.stride[2] % 16 == 0)
    p.slot_body = slot & ~15;
  AppendMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  p.tma_in = 0;
  if (p.run_heads > 0 && es == 2 && (uintptr_t)k.data % 16 == 0 && (uintptr_t)v.data % 16 == 0 &&
      k.stride[0] % 8 == 0 && k.stride[1] % 8 == 0 && v.stride[0] % 8 == 0 &&
      v.stride[1] % 8 == 0 &&
      encode_input_map(&maps.k, k.data, T, h_kv, D, k.stride[0], k.stride[1], p.run_heads,
                       rows / p.run_heads) &&
      encode_input_map(&maps.v, v.data, T, h_kv, D, v.stride[0], v.stride[1], p.run_heads,
                       rows / p.run_heads))
    p.tma_in = 1;
  return launch_append_any(D, k.dtype, p, maps, ds->info, as_stream(stream));
}

tq_status tq_quantize_append_dense(tq_tensor pages, tq_tensor slot_mapping, tq_tensor k,
                                   tq_tensor v, const tq_codebooks* cb, const tq_rotation* rot,
                                   int32_t k_bits, int32_t v_bits, void* stream) {
  if (cb == nullptr) return TQ_ERR_INVALID_ARG;
  if (!valid_tensor(pages, 4) || pages.dtype != TQ_U8 || pages.stride[3] != 1)
    return TQ_ERR_INVALID_ARG;
  if (!valid_tensor(slot_mapping, 1) || slot_mapping.dtype != TQ_I64) return TQ_ERR_INVALID_ARG;
  if (!valid_tensor(k, 3) || !valid_tensor(v, 3) || !is_float_dtype(k.dtype) ||
      k.dtype != v.dtype || k.stride[2] != 1 || v.stride[2] != 1)
    return TQ_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (k.shape[i] != v.shape[i]) return TQ_ERR_INVALID_ARG;
  const int64_t T = k.shape[0];
  const int h_kv = (int)k.shape[1];
  const int D = (int)k.shape[2];
  if (slot_mapping.shape[0] != T || pages.shape[2] != h_kv) return TQ_ERR_INVALID_ARG;
  if (k_bits < 1 || k_bits > 8 || v_bits < 1 || v_bits > 8) return TQ_ERR_INVALID_ARG;
  if (!valid_codebook(cb->k, D) || !valid_codebook(cb->v, D) || cb->k.bits != k_bits ||
      cb->v.bits != v_bits || !valid_rotation(rot, D))
    return TQ_ERR_INVALID_ARG;
  const int kb = region_bytes(D, k_bits), vb = region_bytes(D, v_bits);
  if (pages.shape[3] < kb + vb || pages.shape[3] % 8 != 0) return TQ_ERR_INVALID_ARG;
  if (pages.stride[0] % 4 || pages.stride[1] % 4 || pages.stride[2] % 4 ||
      (uintptr_t)pages.data % 4)
    return TQ_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return TQ_ERR_UNSUPPORTED;
  if (T == 0 || h_kv == 0) return TQ_OK;
  const int box_h = dense_box_heads(h_kv);
  if (box_h == 0 || !dense_input_ok(k) || !dense_input_ok(v)) return TQ_ERR_UNSUPPORTED;
  if (T * h_kv >= ((int64_t)1 << 31) - 256) return TQ_ERR_UNSUPPORTED;
  DeviceState* ds = nullptr;
  tq_status s = device_state(&ds);
  if (s != TQ_OK) return s;
  DenseAppendParams p{};
  p.pages = (uint8_t*)pages.data;
  p.num_slots = pages.shape[0] * pages.shape[1];
  p.block_size = (int32_t)pages.shape[1];
  p.bs_shift = -1;
  for (int sh = 0; sh < 31; ++sh)
    if ((int64_t)1 << sh == pages.shape[1]) p.bs_shift = sh;
  p.h_kv = h_kv;
  p.blk_stride = pages.stride[0];
  p.row_stride = pages.stride[1];
  p.head_stride = pages.stride[2];
  p.slot_mapping = (const int64_t*)slot_mapping.data;
  p.slot_map_stride = slot_mapping.stride[0];
  p.num_tokens = T;
  p.boundaries[0] = cb->k.boundaries;
  p.boundaries[1] = cb->v.boundaries;
  p.bits[0] = k_bits;
  p.bits[1] = v_bits;
  p.rot_hi = rot->hi;
  p.rot_lo = rot->lo;
  p.err = ds->err.load(std::memory_order_relaxed);
  p.box_h = box_h;
  p.wait_ms = kWaitMs;
  DenseAppendMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  if (!encode_input_map(&maps.k, k.data, T, h_kv, D, k.stride[0], k.stride[1], box_h,
                        kDenseRows / box_h) ||
      !encode_input_map(&maps.v, v.data, T, h_kv, D, v.stride[0], v.stride[1], box_h,
                        kDenseRows / box_h))
    return TQ_ERR_UNSUPPORTED;
  return launch_append_dense_any(D, p, maps, ds->info, as_stream(stream));
}

tq_status tq_rotate_unit_dense(tq_tensor u, tq_tensor norm, tq_tensor x, const tq_rotation* rot,
                               void* stream) {
  if (!valid_tensor(x, 2) || !valid_tensor(u, 2) || !valid_tensor(norm, 1)) return TQ_ERR_INVALID_ARG;
  if (x.dtype != TQ_BF16 || u.dtype != TQ_F32 || norm.dtype != TQ_F32) return TQ_ERR_INVALID_ARG;
  if (x.stride[1] != 1 || u.stride[1] != 1 || norm.stride[0] != 1 || u.shape[0] != x.shape[0] ||
      u.shape[1] != x.shape[1] || norm.shape[0] != x.shape[0])
    return TQ_ERR_INVALID_ARG;
  const int D = (int)x.shape[1];
  if (!valid_rotation(rot, D)) return TQ_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return TQ_ERR_UNSUPPORTED;
  if (x.shape[0] == 0) return TQ_OK;
  if ((uintptr_t)x.data % 16 || x.stride[0] % 8 || x.shape[0] >= ((int64_t)1 << 31) - 256)
    return TQ_ERR_UNSUPPORTED;
  DeviceState* ds = nullptr;
  tq_status s = device_state(&ds);
  if (s != TQ_OK) return s;
  DenseAppendParams p{};
  p.num_tokens = x.shape[0];
  p.h_kv = 1;
  p.bits[0] = p.bits[1] = 1;
  p.boundaries[0] = p.boundaries[1] = nullptr;
  p.rot_hi = rot->hi;
  p.rot_lo = rot->lo;
  p.err = ds->err.load(std::memory_order_relaxed);
  p.box_h = 1;
  p.wait_ms = kWaitMs;
  p.export_mode = 1;
  p.u_out = (float*)u.data;
  p.u_stride = u.stride[0];
  p.n_out = (float*)norm.data;
  DenseAppendMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  if (!encode_input_map(&maps.k, x.data, x.shape[0], 1, D, x.stride[0], D, 1, kDenseRows))
    return TQ_ERR_UNSUPPORTED;
  maps.v = maps.k;
  return launch_append_dense_any(D, p, maps, ds->info, as_stream(stream));
}

tq_status tq_paged_decode_dense(tq_tensor out, tq_tensor q, tq_tensor pages,
                                tq_tensor block_table, tq_tensor seq_lens,
                                const tq_codebooks* cb, const tq_rotation* rot, float scale,
                                void* stream) {
  DecodeCall call;
  tq_status s = decode_prepare(out, q, pages, block_table, seq_lens, cb, scale, &call);
  if (s != TQ_OK) return s;
  if (!valid_rotation(rot, (int)q.shape[2])) return TQ_ERR_INVALID_ARG;
  if (call.B == 0) return TQ_OK;
  uint8_t* ws = nullptr;
  s = decode_workspace(call, &ws);
  if (s != TQ_OK) return s;
  return decode_run(call, out, q, pages, block_table, seq_lens, cb, 0, scale, ws, stream,
                    HotWindow(), rot);
}

tq_status tq_decode_plan_probe(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                               int32_t head_dim, int32_t k_bits, int32_t v_bits,
                               int32_t slot_stride, int32_t max_blocks, int32_t num_sms,
                               int32_t max_smem_optin, uint32_t dyn_smem_base, int64_t* out) {
  if (out == nullptr || batch < 1 || num_q_heads < 1 || num_kv_heads < 1 || head_dim < 1 ||
      slot_stride < 1 || max_blocks < 1 || num_sms < 1 || max_smem_optin < 1 ||
      num_q_heads % num_kv_heads)
    return TQ_ERR_INVALID_ARG;
  DeviceInfo di;
  di.num_sms = num_sms;
  di.max_smem_optin = max_smem_optin;
  di.dyn_smem_base = dyn_smem_base;
  DecodePlan plan;
  const tq_status s = plan_decode(batch, num_q_heads, num_kv_heads, head_dim, k_bits, v_bits,
                                  slot_stride, max_blocks, true, di, &plan);
  if (s != TQ_OK) return s;
  const int64_t v[14] = {plan.wph,          plan.nst,          plan.row_pitch, plan.stage_bytes,
                         plan.lut_win,      plan.lut_off,      plan.lut_bytes, plan.stage_lo_off,
                         plan.stage_hi_off, plan.n_low,        plan.misc_off,  (int64_t)plan.smem,
                         plan.copy_mode,    plan.maxw};
  for (int i = 0; i < 14; ++i) out[i] = v[i];
  return TQ_OK;
}

tq_status tq_rotate_unit(tq_tensor u, tq_tensor norm, tq_tensor x, uint64_t sign_seed,
                         void* stream) {
  if (!valid_tensor(x, 2) || !valid_tensor(u, 2) || !valid_tensor(norm, 1)) return TQ_ERR_INVALID_ARG;
  if (!is_float_dtype(x.dtype) || u.dtype != TQ_F32 || norm.dtype != TQ_F32) return TQ_ERR_INVALID_ARG;
  if (x.stride[1] != 1 || u.stride[1] != 1 || u.shape[0] != x.shape[0] ||
      u.shape[1] != x.shape[1] || norm.shape[0] != x.shape[0])
    return TQ_ERR_INVALID_ARG;
  const int D = (int)x.shape[1];
  if (D != 64 && D != 128 && D != 256) return TQ_ERR_UNSUPPORTED;
  if (x.shape[0] == 0) return TQ_OK;
  DeviceState* ds = nullptr;
  tq_status s = device_state(&ds);
  if (s != TQ_OK) return s;
  RotateParams p{};
  p.x = x.data;
  p.x_row_stride = x.stride[0];
  p.rows = x.shape[0];
  p.u = (float*)u.data;
  p.u_row_stride = u.stride[0];
  p.norm = (float*)norm.data;
  p.norm_stride = norm.stride[0];
  p.sign_seed = sign_seed;
  p.align_mode = align_mode_of(x.data, dtype_size(x.dtype), {x.stride[0]});
  if (x.dtype == TQ_F32 && p.align_mode == 0) return TQ_ERR_INVALID_ARG;
  return launch_rotate_any(D, x.dtype, p, ds->info, as_stream(stream));
}

tq_status tq_decode_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                   int32_t head_dim, int32_t max_blocks, int32_t block_size,
                                   size_t* bytes) {
  if (bytes == nullptr || batch < 0 || num_q_heads < 1 || num_kv_heads < 1 || max_blocks < 0 ||
      block_size != kBlockSize || num_q_heads % num_kv_heads)
    return TQ_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  tq_status s = device_state(&ds);
  if (s != TQ_OK) return s;
  // the record area is sized for the largest warps-per-head count, so any bit widths fit
  DecodePlan plan;
  s = plan_decode(std::max(batch, 1), num_q_heads, num_kv_heads, head_dim, 1, 1,
                  region_bytes(head_dim, 1) * 2 + 8, std::max(max_blocks, 1), false, ds->info,
                  &plan);
  if (s != TQ_OK) return s;
  *bytes = plan.ws_bytes;
  return TQ_OK;
}

tq_status tq_set_workspace(void* ptr, size_t bytes) {
  DeviceState* ds = nullptr;
  tq_status s = device_state(&ds);
  if (s != TQ_OK) return s;
  if (ptr != nullptr && (uintptr_t)ptr % 256) return TQ_ERR_INVALID_ARG;
  // the merge counters at the start of a workspace must read zero before first use
  if (ptr != nullptr && cudaMemset(ptr, 0, bytes) != cudaSuccess) return TQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  ds->user_ws = ptr;
  ds->user_ws_bytes = ptr ? bytes : 0;
  return TQ_OK;
}

tq_status tq_get_device_error(int32_t* out, void* stream) {
  if (out == nullptr) return TQ_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  tq_status s = device_state(&ds);
  if (s != TQ_OK) return s;
  cudaStream_t st = as_stream(stream);
  unsigned int h = 0;
  unsigned int* err = ds->err.load(std::memory_order_relaxed);
  if (cudaMemcpyAsync(&h, err, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return TQ_ERR_CUDA;
  if (cudaMemsetAsync(err, 0, sizeof(unsigned int), st) != cudaSuccess) return TQ_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return TQ_ERR_CUDA;
  if (h != 0) {
    // a launch that reported an error may have stopped with merge counters raised:
    // clear the counter areas of this device's workspaces
    std::lock_guard<std::mutex> lock(g_mu);
    const size_t n = ds->counter_bytes;
    if (n > 0) {
      if (ds->user_ws && cudaMemset(ds->user_ws, 0, std::min(n, ds->user_ws_bytes)) != cudaSuccess)
        return TQ_ERR_CUDA;
      if (ds->lib_ws && cudaMemset(ds->lib_ws, 0, std::min(n, ds->lib_ws_bytes)) != cudaSuccess)
        return TQ_ERR_CUDA;
      if (ds->noalloc_scratch &&
          cudaMemset(ds->noalloc_scratch, 0, std::min<size_t>(n, TQ_NOALLOC_SCRATCH_BYTES)) !=
              cudaSuccess)
        return TQ_ERR_CUDA;
    }
  }
  *out = (int32_t)h;
  return TQ_OK;
}

tq_status tq_debug_inject_merge_stall(int32_t withhold_cta, int32_t wait_ms) {
  if (withhold_cta < 0 || wait_ms < 1 || wait_ms > (int32_t)kWaitMs) return TQ_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  tq_status s = device_state(&ds);
  if (s != TQ_OK) return s;
  std::lock_guard<std::mutex> lock(g_mu);
  ds->inject_withhold = withhold_cta;
  ds->inject_wait_ms = (uint32_t)wait_ms;
  return TQ_OK;
}

tq_status tq_paged_decode(tq_tensor out, tq_tensor q, tq_tensor pages, tq_tensor block_table,
                          tq_tensor seq_lens, const tq_codebooks* cb, uint64_t sign_seed,
                          float scale, void* stream) {
  DecodeCall call;
  tq_status s = decode_prepare(out, q, pages, block_table, seq_lens, cb, scale, &call);
  if (s != TQ_OK || call.B == 0) return s;
  uint8_t* ws = nullptr;
  s = decode_workspace(call, &ws);
  if (s != TQ_OK) return s;
  return decode_run(call, out, q, pages, block_table, seq_lens, cb, sign_seed, scale, ws, stream);
}

tq_status tq_paged_decode_qjl(tq_tensor out, tq_tensor q, tq_tensor pages, tq_tensor block_table,
                              tq_tensor seq_lens, const tq_codebooks* cb, uint64_t sign_seed,
                              uint64_t qjl_seed, float scale, void* stream) {
  DecodeCall call;
  tq_status s = decode_prepare(out, q, pages, block_table, seq_lens, cb, scale, &call, true);
  if (s != TQ_OK || call.B == 0) return s;
  uint8_t* ws = nullptr;
  s = decode_workspace(call, &ws);
  if (s != TQ_OK) return s;
  return decode_run(call, out, q, pages, block_table, seq_lens, cb, sign_seed, scale, ws, stream,
                    HotWindow(), nullptr, qjl_seed);
}

tq_status tq_paged_decode_hot(tq_tensor out, tq_tensor q, tq_tensor pages, tq_tensor block_table,
                              tq_tensor seq_lens, tq_tensor hot_k, tq_tensor hot_v,
                              tq_tensor hot_lens, const tq_codebooks* cb, uint64_t sign_seed,
                              float scale, void* stream) {
  DecodeCall call;
  tq_status s = decode_prepare(out, q, pages, block_table, seq_lens, cb, scale, &call);
  if (s != TQ_OK) return s;
  HotWindow hw;
  hw.k = &hot_k;
  hw.v = &hot_v;
  hw.lens = &hot_lens;
  s = hot_validate(call, q, hw);
  if (s != TQ_OK || call.B == 0) return s;
  uint8_t* ws = nullptr;
  s = decode_workspace(call, &ws);
  if (s != TQ_OK) return s;
  return decode_run(call, out, q, pages, block_table, seq_lens, cb, sign_seed, scale, ws, stream,
                    hw);
}

tq_status tq_paged_decode_noalloc(tq_tensor out, tq_tensor q, tq_tensor pages,
                                  tq_tensor block_table, tq_tensor seq_lens,
                                  const tq_codebooks* cb, uint64_t sign_seed, float scale,
                                  void* stream) {
  DecodeCall call;
  tq_status s = decode_prepare(out, q, pages, block_table, seq_lens, cb, scale, &call);
  if (s != TQ_OK || call.B == 0) return s;
  if (call.plan.ws_bytes > TQ_NOALLOC_SCRATCH_BYTES) return TQ_ERR_WORKSPACE;
  DeviceState* ds = call.ds;
  uint8_t* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (ds->noalloc_scratch == nullptr) {
      // one-time set-up on this device (the current one): the scratch array's address
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_tq_noalloc_scratch) != cudaSuccess || addr == nullptr)
        return TQ_ERR_CUDA;
      ds->noalloc_scratch = (uint8_t*)addr;
    }
    ws = ds->noalloc_scratch;
  }
  // The scratch starts zeroed (a static device array) and every call leaves its merge
  // counters at zero; the partial records a launch reads are written earlier in the
  // same launch.
  return decode_run(call, out, q, pages, block_table, seq_lens, cb, sign_seed, scale, ws, stream);
}

}  // extern "C"
