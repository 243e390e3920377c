// tq_decode.cuh -- paged decode attention straight over packed TurboQuant slots.
//
// Follows tq-kv (shadowgraph.io), "Library API" (pre_rotate_query_with_signs, then
// fused_attention_scores on the compressed keys with a scale) and "Custom CUDA Kernel
// Stack" (flash decode v2: split-KV, online softmax; TQ fused attention: scores
// without decompression); turboquant_pro 1.4.2, "Fused CUDA decode" (split-K decode
// computed on the codes, no reconstruction); TorbuQuant, "TQ4 page tensor" (slot ->
// block, row; K region then V region).
//
// Math.  With R the rotation, k_hat_t = nK_t R^T cK[idx_t] and v_hat_t = nV_t R^T cV[.]:
//   <q, k_hat_t> = nK_t <R q, cK[idx_t]>            (score on the codes)
//   sum_t p_t v_hat_t = R^T sum_t p_t nV_t cV[.]       (V in the rotated domain)
// so q is rotated once, and the output is rotated back once (merge kernel).
//
// Kernel layout (one CTA per (sequence, split); one warp per (KV head, sub-stream)):
//   * whole page blocks (16 rows x all KV heads x slot stride, contiguous) are staged
//     into shared memory with cp.async in a multi-stage ring;
//   * codes are turned into fp16 through a per-CTA lookup table of code PAIRS
//     (bits <= 4) or single codes (bits > 4);
//   * S = Qhat . K~^T runs on mma.sync m16n8k16 (M = query heads of the group, N = 16
//     tokens, K = D), fp32 accumulation; the score is s = acc * nK * |q'| * scale;
//   * online softmax in base 2 with a running reference M = max(s + log2 nV), so the
//     fp16 weights P~ = 2^(s - M) nV never exceed 1 (no overflow for large V norms);
//   * O'^T += V~^T . P~^T on mma.sync (M = coordinates, N = query heads, K = tokens):
//     the C fragment of S is exactly the B fragment of this product (no shuffles);
//   * each warp writes its partial (M, l, O') to the workspace; the merge kernel
//     combines the partials, divides by l and applies the inverse rotation.
#pragma once

#include "tq_device.cuh"

namespace tq {

constexpr int kBlockSize = 16;        // tokens per page block (mma N = 16)
constexpr int kDecodeWarps = 8;

struct DecodeParams {
  const uint8_t* pages;
  int32_t num_blocks;
  int32_t h_kv;
  int32_t slot_stride;          // bytes between heads inside a row
  int64_t blk_stride;           // bytes between blocks
  const int32_t* block_table;
  int64_t bt_stride;            // elements between sequences
  int32_t max_blocks;
  const int32_t* seq_lens;
  int32_t batch;
  const void* q;                // [B, H_q, D]
  int64_t q_bstride, q_hstride; // elements
  int32_t q_dtype;
  int32_t h_q;
  int32_t group;                // G = H_q / H_kv
  const float* kc;              // K centroids
  const float* vc;              // V centroids
  int32_t k_region;             // bytes of the K region (offset of V region)
  float scale_log2;             // scale * log2(e)
  uint64_t sign_seed;
  int32_t wph;                  // warps (sub-streams) per KV head
  int32_t spb;                  // blocks per split
  int32_t nsplit;
  float* ws;                    // partials [B][nsplit*wph][H_q][D + 2]
  unsigned int* err;
};

struct MergeParams {
  const float* ws;
  void* out;
  int64_t o_bstride, o_hstride;
  int32_t out_dtype;
  int32_t h_q;
  int32_t nsplit;
  int32_t wph;
  int32_t spb;
  int32_t max_blocks;
  const int32_t* seq_lens;
  uint64_t sign_seed;
};

template <int D>
__host__ __device__ constexpr float inv_sqrt_dim() {
  return D == 64 ? 0.125f : (D == 128 ? 0.08838834764831845f : 0.0625f);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Read `NBITS` bits (a whole number of bytes) of a little-endian bit stream
// starting at byte `p` into words w[0..]; `p` is ALIGN-byte aligned.
template <int NBITS, int ALIGN>
__device__ __forceinline__ void load_bits(uint32_t (&w)[(NBITS + 31) / 32], const uint8_t* p) {
  constexpr int NB = NBITS / 8;
  constexpr int LOW = NB & (-NB);                       // largest power of two dividing NB
  constexpr int VEC = LOW < ALIGN ? LOW : ALIGN;        // widest safe access
  if constexpr (VEC >= 16) {
#pragma unroll
    for (int i = 0; i < NB / 16; ++i) {
      uint4 v = *(const uint4*)(p + 16 * i);
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  } else if constexpr (VEC == 8) {
#pragma unroll
    for (int i = 0; i < NB / 8; ++i) {
      uint2 v = *(const uint2*)(p + 8 * i);
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  } else if constexpr (VEC == 4) {
#pragma unroll
    for (int i = 0; i < NB / 4; ++i) w[i] = *(const uint32_t*)(p + 4 * i);
  } else if constexpr (VEC == 2) {
#pragma unroll
    for (int i = 0; i < (NBITS + 31) / 32; ++i) w[i] = 0u;
#pragma unroll
    for (int i = 0; i < NB / 2; ++i)
      w[i / 2] |= (uint32_t)(*(const uint16_t*)(p + 2 * i)) << (16 * (i & 1));
  } else {
#pragma unroll
    for (int i = 0; i < (NBITS + 31) / 32; ++i) w[i] = 0u;
#pragma unroll
    for (int i = 0; i < NB; ++i) w[i / 4] |= (uint32_t)p[i] << (8 * (i & 3));
  }
}

// Field of LEN bits at bit offset POS of the word array (compile-time positions).
template <int POS, int LEN, int NW>
__device__ __forceinline__ uint32_t field(const uint32_t (&w)[NW]) {
  constexpr int wi = POS >> 5, o = POS & 31;
  constexpr uint32_t mask = LEN >= 32 ? 0xffffffffu : ((1u << LEN) - 1u);
  if constexpr (o + LEN <= 32) {
    return (w[wi] >> o) & mask;
  } else {
    return ((w[wi] >> o) | (w[wi + 1] << (32 - o))) & mask;
  }
}

// Lookup tables in shared memory.  For BITS <= 4: lut holds 2^(2 BITS) half2 entries,
// entry (x | y << BITS) = (c[x], c[y]).  For BITS > 4: 2^BITS halves.
template <int BITS>
struct CodeLut {
  static constexpr bool kPair = BITS <= 4;
  static constexpr int kWords = kPair ? (1 << (2 * BITS)) : (1 << BITS) / 2;
  static __device__ __forceinline__ void build(uint32_t* lut, const float* c, int tid, int nt) {
    if constexpr (kPair) {
      for (int i = tid; i < (1 << (2 * BITS)); i += nt)
        lut[i] = pack_half2(c[i & ((1 << BITS) - 1)], c[i >> BITS]);
    } else {
      for (int i = tid; i < (1 << BITS) / 2; i += nt) lut[i] = pack_half2(c[2 * i], c[2 * i + 1]);
    }
  }
  // half2 (c[x], c[y])
  static __device__ __forceinline__ uint32_t pair(const uint32_t* lut, uint32_t x, uint32_t y) {
    if constexpr (kPair) {
      return lut[x | (y << BITS)];
    } else {
      const uint16_t* h = reinterpret_cast<const uint16_t*>(lut);
      return (uint32_t)h[x] | ((uint32_t)h[y] << 16);
    }
  }
  // half2 for two consecutive codes packed in a 2*BITS field (x low)
  static __device__ __forceinline__ uint32_t pair_field(const uint32_t* lut, uint32_t f) {
    if constexpr (kPair) {
      return lut[f];
    } else {
      return pair(lut, f & ((1u << BITS) - 1u), f >> BITS);
    }
  }
};

template <int D, int KB, int VB, int NH>
struct DecodeGeom {
  static constexpr int KSTEPS = D / 16;       // k-steps of the score product
  static constexpr int CH = D / 4;            // K coords per thread (per token)
  static constexpr int CV = D / 8;            // V coords per thread
  static constexpr int MT = D / 16;           // m-tiles of the PV product
  static constexpr int KCH_BITS = CH * KB;
  static constexpr int VCH_BITS = CV * VB;
  static constexpr int KPACK = (D * KB + 7) / 8;   // packed bytes of K (norm follows)
  static constexpr int VPACK = (D * VB + 7) / 8;
};

// Per-CTA shared memory layout (bytes):
//   [lutK | lutV | qrot (heads x D fp32) | stages]
template <int D, int KB, int VB>
struct DecodeSmem {
  static constexpr int kLutK = CodeLut<KB>::kWords * 4;
  static constexpr int kLutV = CodeLut<VB>::kWords * 4;
  static constexpr int kLutBytes = ((kLutK + kLutV + 127) / 128) * 128;
};

template <int NSTAGE>
__device__ __forceinline__ bool block_ok(const DecodeParams& p, int b, int blk_idx, int seq_len,
                                         int32_t* blk_out) {
  if (blk_idx * kBlockSize >= seq_len) return false;
  const int32_t blk = p.block_table[(int64_t)b * p.bt_stride + blk_idx];
  *blk_out = blk;
  return blk >= 0 && blk < p.num_blocks;
}

template <int D, int KB, int VB, int NH, int NSTAGE>
__global__ void __launch_bounds__(kDecodeWarps * 32)
decode_kernel(DecodeParams p) {
  using GM = DecodeGeom<D, KB, VB, NH>;
  using LK = CodeLut<KB>;
  using LV = CodeLut<VB>;
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* lutK = (uint32_t*)smem;
  uint32_t* lutV = lutK + LK::kWords;
  float* qrot = (float*)(smem + DecodeSmem<D, KB, VB>::kLutBytes);
  const int heads_cta = p.h_q;                         // all query heads of the sequence
  uint8_t* stages = (uint8_t*)(qrot + heads_cta * D);
  stages = (uint8_t*)(((uintptr_t)stages + 127) & ~(uintptr_t)127);
  const int block_bytes = kBlockSize * p.h_kv * p.slot_stride;
  const int stage_bytes = block_bytes * p.wph;

  const int split = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int nthreads = blockDim.x;

  int seq_len = p.seq_lens[b];
  const int cap = p.max_blocks * kBlockSize;
  if (seq_len < 0 || seq_len > cap) {
    if (split == 0 && tid == 0) report_error(p.err, TQ_DEVERR_SEQLEN_RANGE);
    return;   // the merge kernel writes 0 for this sequence
  }
  const int nblk_seq = (seq_len + kBlockSize - 1) / kBlockSize;
  const int blk_begin = split * p.spb;
  if (blk_begin >= nblk_seq) return;                   // split past the end: no partial
  const int blk_end = min(nblk_seq, blk_begin + p.spb);
  const int nsteps = (blk_end - blk_begin + p.wph - 1) / p.wph;

  // ---- tables and the rotated query (sign flips, FWHT, kept in fp32) ----
  LK::build(lutK, p.kc, tid, nthreads);
  LV::build(lutV, p.vc, tid, nthreads);
  for (int i = tid; i < heads_cta * D; i += nthreads) {
    const int h = i / D, j = i - h * D;
    float x;
    const int64_t off = (int64_t)b * p.q_bstride + (int64_t)h * p.q_hstride + j;
    if (p.q_dtype == TQ_F32) x = ((const float*)p.q)[off];
    else if (p.q_dtype == TQ_BF16) x = __bfloat162float(((const __nv_bfloat16*)p.q)[off]);
    else x = __half2float(((const __half*)p.q)[off]);
    qrot[i] = __uint_as_float(__float_as_uint(x) ^ sign_mask_at(p.sign_seed, j));
  }
  __syncthreads();
  for (int hstep = 1; hstep < D; hstep <<= 1) {
    for (int i = tid; i < heads_cta * D / 2; i += nthreads) {
      const int h = i / (D / 2), k = i - h * (D / 2);
      const int lo = (k / hstep) * 2 * hstep + (k % hstep);
      float* r = qrot + h * D;
      const float a = r[lo], c = r[lo + hstep];
      r[lo] = a + c;
      r[lo + hstep] = a - c;
    }
    __syncthreads();
  }

  // ---- pipeline prologue ----
  const int active_warps = p.h_kv * p.wph;
  auto issue = [&](int step) {
    if (step < nsteps) {
      uint8_t* dst = stages + (step % NSTAGE) * stage_bytes;
      for (int sub = 0; sub < p.wph; ++sub) {
        const int bi = blk_begin + step * p.wph + sub;
        int32_t blk;
        if (bi < blk_end && block_ok<NSTAGE>(p, b, bi, seq_len, &blk)) {
          const uint8_t* src = p.pages + (int64_t)blk * p.blk_stride;
          uint8_t* d = dst + sub * block_bytes;
          for (int c = tid; c < block_bytes / 16; c += nthreads) cp_async16(d + 16 * c, src + 16 * c);
        }
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int s = 0; s < NSTAGE - 1; ++s) issue(s);

  // ---- per-warp constants ----
  const bool warp_active = warp < active_warps;
  const int kvh = warp % p.h_kv;
  const int sub = warp / p.h_kv;
  const int G = p.group;
  // A fragments of Qhat (rows = query heads of this KV head, cols = coords, permuted):
  // k-step ks, thread (gid, tig) holds head gid (and gid+8), coords tig*CH + 4ks + {0..3}.
  uint32_t qa[GM::KSTEPS][4];
  float qscale[2] = {0.f, 0.f};
  if (warp_active) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int g = gid + 8 * hh;
      if (hh < NH && g < G) {
        const float* r = qrot + (kvh * G + g) * D;
        float ss = 0.f;
        for (int j = 0; j < D; ++j) ss = fmaf(r[j], r[j], ss);
        const float nrm = sqrtf(ss);
        const float inv = nrm > 0.f ? 1.0f / nrm : 0.f;
        // |q'| of the orthonormal rotation is |H (s q)| / sqrt(D)
        qscale[hh] = nrm * inv_sqrt_dim<D>() * p.scale_log2;
#pragma unroll
        for (int ks = 0; ks < GM::KSTEPS; ++ks) {
          const int c0 = tig * GM::CH + 4 * ks;
          qa[ks][hh] = pack_half2(r[c0] * inv, r[c0 + 1] * inv);
          qa[ks][hh + 2] = pack_half2(r[c0 + 2] * inv, r[c0 + 3] * inv);
        }
      } else {
#pragma unroll
        for (int ks = 0; ks < GM::KSTEPS; ++ks) { qa[ks][hh] = 0u; qa[ks][hh + 2] = 0u; }
      }
    }
  }

  // running state: heads gid (and gid+8 when NH == 2)
  float Mrun[NH], lrun[NH];
#pragma unroll
  for (int hh = 0; hh < NH; ++hh) { Mrun[hh] = -INFINITY; lrun[hh] = 0.f; }
  float acc[NH][GM::MT][4];
#pragma unroll
  for (int n = 0; n < NH; ++n)
#pragma unroll
    for (int mt = 0; mt < GM::MT; ++mt)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[n][mt][k] = 0.f;

  for (int step = 0; step < nsteps; ++step) {
    cp_async_wait<NSTAGE - 2>();
    __syncthreads();
    issue(step + NSTAGE - 1);
    const int bi = blk_begin + step * p.wph + sub;
    int32_t blk = 0;
    if (!warp_active || bi >= blk_end) continue;
    if (!block_ok<NSTAGE>(p, b, bi, seq_len, &blk)) {
      if (lane == 0) report_error(p.err, TQ_DEVERR_BLOCK_RANGE);
      continue;
    }
    const int valid = min(kBlockSize, seq_len - bi * kBlockSize);
    const uint8_t* blkp = stages + (step % NSTAGE) * stage_bytes + sub * block_bytes;
    auto slot = [&](int row) { return blkp + (row * p.h_kv + kvh) * p.slot_stride; };

    // ---- S = Qhat . K~^T : two n-tiles of 8 tokens (gid and gid + 8) ----
    float sacc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int k = 0; k < 4; ++k) sacc[nt][k] = 0.f;
      uint32_t kw[(GM::KCH_BITS + 31) / 32];
      load_bits<GM::KCH_BITS, 8>(kw, slot(gid + 8 * nt) + tig * (GM::KCH_BITS / 8));
      static_for<GM::KSTEPS>([&](auto KS) {
        constexpr int ks = decltype(KS)::value;
        const uint32_t b0 = LK::pair_field(lutK, field<(4 * ks) * KB, 2 * KB>(kw));
        const uint32_t b1 = LK::pair_field(lutK, field<(4 * ks + 2) * KB, 2 * KB>(kw));
        mma_16816(sacc[nt], qa[ks], b0, b1);
      });
    }
    // tokens held: nt*8 + 2*tig + {0,1}; heads gid (regs 0,1) and gid+8 (regs 2,3)
    float nK[4], nV[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = (i >> 1) * 8 + 2 * tig + (i & 1);
      const uint8_t* s = slot(row);
      nK[i] = *(const float*)(s + GM::KPACK);
      nV[i] = *(const float*)(s + p.k_region + GM::VPACK);
    }
    uint32_t pb[NH][2];
#pragma unroll
    for (int hh = 0; hh < NH; ++hh) {
      float sv[4], zv[4];
      float zmax = -INFINITY;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = (i >> 1) * 8 + 2 * tig + (i & 1);
        const float a = sacc[i >> 1][(i & 1) + 2 * hh];
        const bool ok = row < valid;
        sv[i] = ok ? a * nK[i] * qscale[hh] : -INFINITY;
        // zero norms are clamped; a NaN norm stays NaN and poisons the output
        const float nvc = nV[i] < 1e-30f ? 1e-30f : nV[i];
        zv[i] = ok ? sv[i] + __log2f(nvc) : -INFINITY;
        zmax = fmaxf(zmax, zv[i]);
      }
      zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, 1));
      zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, 2));
      const float Mnew = fmaxf(Mrun[hh], zmax);
      const float alpha = (Mnew == -INFINITY) ? 1.f : exp2f(Mrun[hh] - Mnew);
      float lsum = 0.f, pv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float e = (sv[i] == -INFINITY) ? 0.f : exp2f(sv[i] - Mnew);
        lsum += e;
        pv[i] = (sv[i] == -INFINITY) ? 0.f : exp2f(zv[i] - Mnew);
      }
      lrun[hh] = lrun[hh] * alpha + lsum;
      Mrun[hh] = Mnew;
      // B fragment of P~^T for heads gid (+8 hh): tokens 2tig,2tig+1 | 2tig+8,2tig+9
      pb[hh][0] = pack_half2(pv[0], pv[1]);
      pb[hh][1] = pack_half2(pv[2], pv[3]);
      // rescale accumulators: columns are heads 2tig, 2tig+1 (+8 hh)
      const float a0 = __shfl_sync(0xffffffffu, alpha, (2 * tig) * 4);
      const float a1 = __shfl_sync(0xffffffffu, alpha, (2 * tig + 1) * 4);
#pragma unroll
      for (int mt = 0; mt < GM::MT; ++mt) {
        acc[hh][mt][0] *= a0; acc[hh][mt][1] *= a1;
        acc[hh][mt][2] *= a0; acc[hh][mt][3] *= a1;
      }
    }
    // ---- O'^T += V~^T . P~^T ----
    {
      uint32_t vw[4][(GM::VCH_BITS + 31) / 32];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = (i >> 1) * 8 + 2 * tig + (i & 1);
        load_bits<GM::VCH_BITS, 4>(vw[i], slot(row) + p.k_region + gid * (GM::VCH_BITS / 8));
      }
      static_for<GM::MT>([&](auto MTI) {
        constexpr int mt = decltype(MTI)::value;
        constexpr int c0 = (2 * mt) * VB, c1 = (2 * mt + 1) * VB;
        uint32_t a[4];
        // coords 2mt (rows gid) and 2mt+1 (rows gid+8) of this thread's V chunk;
        // tokens 2tig, 2tig+1 (a[0], a[1]) and 2tig+8, 2tig+9 (a[2], a[3])
        a[0] = LV::pair(lutV, field<c0, VB>(vw[0]), field<c0, VB>(vw[1]));
        a[1] = LV::pair(lutV, field<c1, VB>(vw[0]), field<c1, VB>(vw[1]));
        a[2] = LV::pair(lutV, field<c0, VB>(vw[2]), field<c0, VB>(vw[3]));
        a[3] = LV::pair(lutV, field<c1, VB>(vw[2]), field<c1, VB>(vw[3]));
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) mma_16816(acc[hh][mt], a, pb[hh][0], pb[hh][1]);
      });
    }
  }
  cp_async_wait<0>();

  if (!warp_active) return;
  // ---- write the partial (M, l, O') of every query head of this warp ----
  const int part = split * p.wph + sub;
  float* base = p.ws + ((int64_t)b * p.nsplit * p.wph + part) * (int64_t)p.h_q * (D + 2);
#pragma unroll
  for (int hh = 0; hh < NH; ++hh) {
    float l = lrun[hh];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const int g = gid + 8 * hh;
    if (tig == 0 && g < G) {
      float* rec = base + (int64_t)(kvh * G + g) * (D + 2);
      rec[0] = Mrun[hh];
      rec[1] = l;
    }
#pragma unroll
    for (int mt = 0; mt < GM::MT; ++mt) {
      const int coord = gid * GM::CV + 2 * mt;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int g2 = 8 * hh + 2 * tig + (k & 1);
        const int c = coord + (k >> 1);
        if (g2 < G) base[(int64_t)(kvh * G + g2) * (D + 2) + 2 + c] = acc[hh][mt][k];
      }
    }
  }
}

// Merge the split partials of one (sequence, query head), then o = R^T (O' / l):
// a FWHT of the rotated-domain output, sign flips and the 1/sqrt(D) scale.
template <int D>
__global__ void __launch_bounds__(D)
merge_kernel(MergeParams p) {
  __shared__ float buf[D];
  __shared__ float wts[2];
  const int h = blockIdx.x, b = blockIdx.y, j = threadIdx.x;
  int seq_len = p.seq_lens[b];
  if (seq_len < 0 || seq_len > p.max_blocks * kBlockSize) seq_len = 0;
  const int nblk = (seq_len + kBlockSize - 1) / kBlockSize;
  const int nsplit_used = (nblk + p.spb - 1) / p.spb;
  const int nparts = nsplit_used * p.wph;
  const float* base = p.ws + (int64_t)b * p.nsplit * p.wph * p.h_q * (D + 2) + (int64_t)h * (D + 2);
  const int64_t pstride = (int64_t)p.h_q * (D + 2);
  float M = -INFINITY;
  for (int i = 0; i < nparts; ++i) M = fmaxf(M, base[i * pstride]);
  float o = 0.f, l = 0.f;
  if (M != -INFINITY) {
    for (int i = 0; i < nparts; ++i) {
      const float* rec = base + i * pstride;
      const float mi = rec[0];
      if (mi == -INFINITY) continue;
      const float w = exp2f(mi - M);
      l += w * rec[1];
      o += w * rec[2 + j];
    }
  }
  buf[j] = (l > 0.f) ? o / l : 0.f;
  (void)wts;
  __syncthreads();
  for (int hs = 1; hs < D; hs <<= 1) {
    float v = 0.f;
    const int partner = j ^ hs;
    const float mine = buf[j], other = buf[partner];
    v = (j & hs) ? other - mine : mine + other;
    __syncthreads();
    buf[j] = v;
    __syncthreads();
  }
  float r = buf[j] * inv_sqrt_dim<D>();
  r = __uint_as_float(__float_as_uint(r) ^ sign_mask_at(p.sign_seed, j));
  const int64_t off = (int64_t)b * p.o_bstride + (int64_t)h * p.o_hstride + j;
  if (p.out_dtype == TQ_F32) ((float*)p.out)[off] = r;
  else if (p.out_dtype == TQ_BF16) ((__nv_bfloat16*)p.out)[off] = __float2bfloat16(r);
  else ((__half*)p.out)[off] = __float2half(r);
}

}  // namespace tq
