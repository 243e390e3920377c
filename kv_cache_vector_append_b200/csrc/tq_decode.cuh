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
// Kernel layout.  A prep kernel rotates every query once.  The decode kernel is
// persistent: the (sequence, pair of blocks) steps of the whole batch are laid end
// to end and CTA c takes the equal contiguous range [c S/C, (c+1) S/C) of the S
// steps (stream-K style), so ragged batches and single long sequences balance
// alike.  Inside a CTA one warp serves one (KV head, sub-stream):
//   * page blocks (16 tokens x all KV heads; one per sub-stream and step) are staged
//     into shared memory by one TMA tensor copy each (a 16-row box one padding wider
//     than a row, the padding zero-filled out of bounds) into a 4-deep ring of stages
//     guarded by mbarriers; the last warp to release a stage refills it, so no warp
//     ever waits for the whole CTA; the padded pitch of 20 (mod 32) words makes the
//     per-thread code loads below bank-conflict free;
//   * codes become fp16 through per-lane replicated lookup tables of code PAIRS
//     (bits <= 4: entry (x | y << bits) = (c[x], c[y])) or single codes, so that
//     the 32 lanes of a warp always hit 32 different banks;
//   * S^T = K~ . Qhat^T on mma.sync m16n8k16 (M = 16 tokens, N = 8 query heads of the
//     group, K = D; fp16 operands, fp32 accumulation); s = acc * nK * |q'| * scale * log2 e;
//   * online softmax in base 2 against a running reference M >= max(s + e(nV)),
//     e(x) = floor(log2 x) + 1 read from the exponent bits, raised only when a tile
//     exceeds it by more than 2^8 (lazy rescale), so the fp16 weights
//     P~ = 2^(s - M) nV stay below 2^9 whatever the V norms;
//   * O'^T += V~^T . P~^T on mma.sync (M = coordinates, N = query heads, K = tokens);
//     the fp16 weights go from the C layout of S^T to the B layout of P~^T with one
//     movmatrix transpose per 8 x 8 tile;
//   * at every sequence boundary of its range a warp writes its partial (M, l, O')
//     to record (CTA + sequence), an index no other (CTA, sequence) pair shares
//     because the ranges are monotone; the merge kernel combines the records of a
//     sequence, divides by l and applies the inverse rotation.
// The coordinate order inside each mma tile is free (a permutation applied to both
// operands of a contraction leaves it unchanged); it is chosen so that every thread
// reads whole 32-bit words of codes, and undone when O' is written out.
#pragma once

#include "tq_device.cuh"

namespace tq {

constexpr int kBlockSize = 16;        // tokens per page block
constexpr int kDecodeWarps = 8;
constexpr int kDecodeStages = 4;
constexpr uint32_t kWaitLimit = 2000;      // polls (each <= ~1 ms) before a wait gives up
constexpr float kLazyRescale = 8.0f;  // log2 units

struct DecodeParams {
  const uint8_t* pages;
  int32_t num_blocks;
  int32_t h_kv;
  int32_t slot_stride;          // bytes between heads inside a row
  int32_t row_pitch;            // bytes between rows in shared memory (padded)
  int64_t blk_stride;           // bytes between blocks in global memory
  const int32_t* block_table;
  int64_t bt_stride;            // elements between sequences
  int32_t max_blocks;
  const int32_t* seq_lens;
  int32_t batch;
  int32_t h_q;
  int32_t group;                // G = H_q / H_kv
  const float* kc;              // K centroids
  const float* vc;              // V centroids
  int32_t shared_lut;           // K and V tables identical (one LUT)
  int32_t k_region;             // bytes of the K region (offset of V region)
  int32_t wph;                  // warps (sub-streams) per KV head = blocks per step
  int32_t stage_bytes;
  int32_t ids_cap;              // block ids of its step range a CTA preloads (entries)
  int32_t copy_mode;            // 1: 2-D tensor box per block (rows padded to row_pitch)
                                // 0: 1-D bulk copy per block (row_pitch = row bytes)
  const uint32_t* qfrag;        // [B][H_q][4 tig][KSTEPS][2] half2, from qprep_kernel
  const float* qscale;          // [B][H_q]: |q'| * scale * log2(e)
  int32_t* prefix;              // [B + 1] step prefix sums (written by CTA 0)
  float* part;                  // records [(C + B)][wph][H_q][D + 2]
  unsigned int* err;
};

struct QPrepParams {
  const void* q;                // [B, H_q, D]
  int64_t q_bstride, q_hstride; // elements
  int32_t q_dtype;
  int32_t h_q;
  float scale_log2;             // scale * log2(e)
  uint64_t sign_seed;
  uint32_t* qfrag;
  float* qscale;
};

struct MergeParams {
  const float* part;
  const int32_t* prefix;
  void* out;
  int64_t o_bstride, o_hstride;
  int32_t out_dtype;
  int32_t h_q;
  int32_t wph;
  int32_t nctas;
  uint64_t sign_seed;
};

// Step range of CTA c out of C over S steps: [floor(c S / C), floor((c+1) S / C)).
__host__ __device__ __forceinline__ int64_t cta_begin(int64_t c, int64_t S, int64_t C) {
  return c * S / C;
}
// The CTA whose range holds step x: the largest c with cta_begin(c) <= x.
__host__ __device__ __forceinline__ int64_t cta_of(int64_t x, int64_t S, int64_t C) {
  return ((x + 1) * C - 1) / S;
}

template <int D>
__host__ __device__ constexpr float inv_sqrt_dim() {
  return D == 64 ? 0.125f : (D == 128 ? 0.08838834764831845f : 0.0625f);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Field of LEN bits at bit offset POS of a word (compile-time position); whole bytes
// are extracted with one byte permute.
template <int POS, int LEN>
__device__ __forceinline__ uint32_t bits_of(uint32_t w) {
  constexpr uint32_t mask = LEN >= 32 ? 0xffffffffu : ((1u << LEN) - 1u);
  if constexpr (LEN == 8 && POS % 8 == 0) {
    return __byte_perm(w, 0u, 0x4440u | (POS / 8));
  } else if constexpr (POS + LEN == 32) {
    return w >> POS;
  } else {
    return (w >> POS) & mask;
  }
}

// Field of LEN bits at bit offset POS of the word array (compile-time positions).
template <int POS, int LEN, int NW>
__device__ __forceinline__ uint32_t field(const uint32_t (&w)[NW]) {
  constexpr int wi = POS >> 5, o = POS & 31;
  constexpr uint32_t mask = LEN >= 32 ? 0xffffffffu : ((1u << LEN) - 1u);
  if constexpr (o + LEN <= 32) {
    return bits_of<o, LEN>(w[wi]);
  } else {
    return ((w[wi] >> o) | (w[wi + 1] << (32 - o))) & mask;
  }
}

// How one thread's share of a packed region is read.  A region of NWORDS words
// holds D codes of BITS bits; NT threads split it, each taking D/NT codes:
//   kInterleaved: thread t reads words t, t+NT, t+2NT, ... (codes never straddle
//                 words when 32 % BITS == 0); conflict free with the padded pitch;
//   kContig:      thread t reads NWORDS/NT consecutive words;
//   kBytes:       thread t reads its (D/NT)*BITS/8 bytes one by one.
// Code m of the thread's list sits at bit pos(m) of the loaded word array and is
// coordinate coord(t, m) of the row.
template <int D, int BITS, int NT>
struct Share {
  static constexpr int NCODES = D / NT;
  static constexpr int NWORDS = D * BITS / 32;
  static constexpr bool kInterleaved = (32 % BITS == 0) && (NWORDS % NT == 0);
  static constexpr bool kContig = !kInterleaved && (NWORDS % NT == 0);
  static constexpr int PW = 32 / BITS;                   // codes per word (interleaved)
  static constexpr int NW = kInterleaved || kContig ? NWORDS / NT : (NCODES * BITS + 31) / 32;
  static constexpr int BYTES = NCODES * BITS / 8;        // kBytes: bytes per thread

  static __host__ __device__ constexpr int pos(int m) {
    return kInterleaved ? 32 * (m / PW) + (m % PW) * BITS : m * BITS;
  }
  static __host__ __device__ constexpr int coord(int t, int m) {
    return kInterleaved ? (t + NT * (m / PW)) * PW + (m % PW) : t * NCODES + m;
  }
  // region: 4-byte aligned start of the packed codes
  static __device__ __forceinline__ void load(uint32_t (&w)[NW], const uint8_t* region, int t) {
    if constexpr (kInterleaved) {
#pragma unroll
      for (int j = 0; j < NW; ++j) w[j] = *(const uint32_t*)(region + 4 * (t + NT * j));
    } else if constexpr (kContig) {
#pragma unroll
      for (int j = 0; j < NW; ++j) w[j] = *(const uint32_t*)(region + 4 * (NW * t + j));
    } else {
#pragma unroll
      for (int j = 0; j < NW; ++j) w[j] = 0u;
      const uint8_t* p = region + BYTES * t;
#pragma unroll
      for (int i = 0; i < BYTES; ++i) w[i / 4] |= (uint32_t)p[i] << (8 * (i & 3));
    }
  }
};

// Replicated lookup tables.  Entry e of the table for lane l is the 32-bit word at
// index (e << 5) | l, so lookups by a warp never conflict.  For BITS <= 4 the
// table holds code pairs: entry (x | y << BITS) = half2(c[x], c[y]); for BITS > 4
// it holds single codes: entry x = half2(c[x], c[x]).
template <int BITS>
struct RepLut {
  static constexpr bool kPair = BITS <= 4;
  static constexpr int kEntries = kPair ? (1 << (2 * BITS)) : (1 << BITS);
  static constexpr int kBytes = kEntries * 32 * 4;
  // c: the 2^BITS centroids, already in shared memory
  static __device__ __forceinline__ void build(uint32_t* lut, const float* c, int tid, int nt) {
    for (int i = tid; i < kEntries * 32; i += nt) {
      const int e = i >> 5;
      if constexpr (kPair) lut[i] = pack_half2(c[e & ((1 << BITS) - 1)], c[e >> BITS]);
      else lut[i] = pack_half2(c[e], c[e]);
    }
  }
  // half2 (c[x], c[y]); `lane_lut` = lut + lane
  static __device__ __forceinline__ uint32_t pair(const uint32_t* lane_lut, uint32_t x,
                                                  uint32_t y) {
    if constexpr (kPair) {
      return lane_lut[(x | (y << BITS)) << 5];
    } else {
      const uint32_t lo = lane_lut[x << 5], hi = lane_lut[y << 5];
      return __byte_perm(lo, hi, 0x7610);   // low half of lo, high half of hi
    }
  }
  // pair packed in one 2*BITS field (x in the low bits)
  static __device__ __forceinline__ uint32_t pair_field(const uint32_t* lane_lut, uint32_t f) {
    if constexpr (kPair) return lane_lut[f << 5];
    else return pair(lane_lut, f & ((1u << BITS) - 1u), f >> BITS);
  }
};

// Transpose of an 8x8 matrix of 16-bit values held in mma fragment layout.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
  return d;
}

template <int D, int KB, int VB>
struct DecodeCfg {
  using KS = Share<D, KB, 4>;     // K: 4 threads (tig) per token row
  using VS = Share<D, VB, 8>;     // V: 8 threads (gid) per token row
  static constexpr int KSTEPS = D / 16;
  static constexpr int MT = D / 16;
  static constexpr int KPACK = D * KB / 8;   // packed bytes (the norm follows)
  static constexpr int VPACK = D * VB / 8;
  static constexpr int kLutBytes = RepLut<KB>::kBytes + RepLut<VB>::kBytes;
};

// q' = R q for every (sequence, query head): sign flips, FWHT, 1/sqrt(D); stored as
// q'/|q'| in fp16, already in the A-fragment order of the score product (thread
// tig, k-step ks: coords KS::coord(tig, 4ks .. 4ks+3)), and |q'| * scale * log2 e.
// One warp per (sequence, query head): each lane holds D/32 consecutive coordinates,
// the FWHT runs in registers and across lanes with shuffles.
template <int D, int KB>
__global__ void __launch_bounds__(256)
qprep_kernel(QPrepParams p, int32_t rows) {
  using KS = Share<D, KB, 4>;
  constexpr int E = D / 32;
  constexpr int NWORDS = D / 2;          // fragment words per head
  __shared__ float sbuf[8][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;   // = b * H_q + h
  if (row >= rows) return;
  const int b = row / p.h_q, h = row - b * p.h_q;
  float x[E];
  const int64_t off = (int64_t)b * p.q_bstride + (int64_t)h * p.q_hstride + lane * E;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    float v;
    if (p.q_dtype == TQ_F32) v = ((const float*)p.q)[off + e];
    else if (p.q_dtype == TQ_BF16) v = __bfloat162float(((const __nv_bfloat16*)p.q)[off + e]);
    else v = __half2float(((const __half*)p.q)[off + e]);
    x[e] = __uint_as_float(__float_as_uint(v) ^ sign_mask_at(p.sign_seed, lane * E + e));
  }
#pragma unroll
  for (int hs = 1; hs < E; hs <<= 1)
#pragma unroll
    for (int i = 0; i < E; ++i)
      if ((i & hs) == 0) {
        const float a = x[i], c = x[i + hs];
        x[i] = a + c;
        x[i + hs] = a - c;
      }
#pragma unroll
  for (int lm = 1; lm < 32; lm <<= 1)
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, x[i], lm);
      x[i] = (lane & lm) ? o - x[i] : x[i] + o;
    }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    x[i] *= inv_sqrt_dim<D>();
    ss = fmaf(x[i], x[i], ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float nrm = sqrtf(ss);
  const float inv = nrm > 0.f ? 1.0f / nrm : 0.f;
#pragma unroll
  for (int i = 0; i < E; ++i) sbuf[warp][lane * E + i] = x[i] * inv;
  __syncwarp();
  uint32_t* dst = p.qfrag + (int64_t)row * NWORDS;
  for (int w = lane; w < NWORDS; w += 32) {
    // word w = (tig, ks, hi): codes 4ks + 2hi, +1 of thread tig's share
    const int tig = w / (NWORDS / 4), ks = (w / 2) % (D / 16), hi = w & 1;
    const int m0 = 4 * ks + 2 * hi;
    int c0, c1;
    if constexpr (KS::kInterleaved) {
      c0 = (tig + 4 * (m0 / KS::PW)) * KS::PW + (m0 % KS::PW);
      c1 = (tig + 4 * ((m0 + 1) / KS::PW)) * KS::PW + ((m0 + 1) % KS::PW);
    } else {
      c0 = tig * KS::NCODES + m0;
      c1 = c0 + 1;
    }
    dst[w] = pack_half2(sbuf[warp][c0], sbuf[warp][c1]);
  }
  if (lane == 0) p.qscale[row] = nrm * p.scale_log2;
}

// floor(log2 x) + 1 for x > 0 (exponent bits; an upper bound of log2 x within 1),
// -126 for zero or subnormal x, NaN for NaN.
__device__ __forceinline__ float log2_ceilish(float x) {
  const uint32_t e = (__float_as_uint(x) >> 23) & 0xFFu;
  const float f = __uint_as_float(0x4B000000u | e) - 8388608.0f;   // exact small integer
  return x != x ? x : f - 126.0f;
}

// Shared memory: [K LUT | V LUT | stages | full mbarriers | release counters | prefix |
// centroids].
template <int D, int KB, int VB, int NH>
__global__ void __launch_bounds__(kDecodeWarps * 32, (NH == 1 && D <= 128) ? 2 : 1)
decode_kernel(DecodeParams p, const __grid_constant__ CUtensorMap tmap) {
  using C = DecodeCfg<D, KB, VB>;
  using KS = typename C::KS;
  using VS = typename C::VS;
  using LK = RepLut<KB>;
  using LV = RepLut<VB>;
  constexpr int NST = kDecodeStages;
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* lutK = (uint32_t*)smem;
  const bool one_lut = KB == VB && p.shared_lut;
  uint32_t* lutV = one_lut ? lutK : lutK + LK::kBytes / 4;
  uint8_t* stages = smem + (one_lut ? LK::kBytes : C::kLutBytes);
  stages += (128u - (smem_u32(stages) & 127u)) & 127u;   // TMA destinations: 128-byte aligned
  uint64_t* full = (uint64_t*)(stages + NST * p.stage_bytes);
  int* released = (int*)(full + NST);
  uint32_t* present = (uint32_t*)(released + NST);     // per stage: bit k = block k staged
  int32_t* prefix = (int32_t*)(present + NST);
  float* cents = (float*)(prefix + p.batch + 1);   // K centroids, then V centroids
  int32_t* ids = (int32_t*)(cents + (1 << KB) + (1 << VB));   // block ids of the range

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int nthreads = blockDim.x;
  const int nwarps = nthreads >> 5;                    // = h_kv * wph
  const int per_step = p.wph;                          // blocks per pipeline step

  // ---- step prefix sums over the sequences (every CTA; CTA 0 publishes them) ----
  {
    __shared__ int s_part[kDecodeWarps * 32];
    const int B = p.batch;
    const int chunk = (B + nthreads - 1) / nthreads;
    const int lo = tid * chunk, hi = min(B, lo + chunk);
    int sum = 0;
    for (int b = lo; b < hi; ++b) {
      const int len = p.seq_lens[b];
      int steps = 0;
      if (len < 0 || len > p.max_blocks * kBlockSize) {
        if (blockIdx.x == 0) report_error(p.err, TQ_DEVERR_SEQLEN_RANGE);
      } else {
        steps = ((len + kBlockSize - 1) / kBlockSize + per_step - 1) / per_step;
      }
      prefix[b + 1] = steps;
      sum += steps;
    }
    s_part[tid] = sum;
    if (tid < NST) {
      mbar_init(&full[tid], 1);
      released[tid] = 0;
    }
    for (int i = tid; i < (1 << KB); i += nthreads) cents[i] = p.kc[i];
    for (int i = tid; i < (1 << VB); i += nthreads) cents[(1 << KB) + i] = p.vc[i];
    fence_mbar_init();
    __syncthreads();
    if (tid == 0) {
      int run = 0;
      for (int t = 0; t < nthreads; ++t) { const int v = s_part[t]; s_part[t] = run; run += v; }
      prefix[0] = 0;
    }
    __syncthreads();
    int run = s_part[tid];
    for (int b = lo; b < hi; ++b) { run += prefix[b + 1]; prefix[b + 1] = run; }
    __syncthreads();
    if (blockIdx.x == 0)
      for (int b = tid; b <= B; b += nthreads) p.prefix[b] = prefix[b];
  }
  const int64_t S = prefix[p.batch];
  const int64_t Cn = gridDim.x;
  const int64_t s0 = cta_begin(blockIdx.x, S, Cn), s1 = cta_begin(blockIdx.x + 1, S, Cn);
  if (s0 >= s1) return;
  // sequence walk: the largest b with prefix[b] <= s, then advance step by step
  auto locate = [&](int64_t s) {
    int lo = 0, hi = p.batch;           // prefix[lo] <= s < prefix[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= s) lo = mid; else hi = mid;
    }
    return lo;
  };

  const int pitch = p.row_pitch;
  const int blk_smem = kBlockSize * pitch;
  const int row_bytes = p.h_kv * p.slot_stride;
  // Block id of block k of global step s: -1 past the end of its sequence or when the
  // table entry is out of range (reported).  The ids of the whole step range are
  // preloaded into shared memory below (up to ids_cap of them) so that a refill never
  // waits on a global load.
  auto block_id = [&](int64_t s, int k) -> int32_t {
    const int b = locate(s);
    const int bi = (int)(s - prefix[b]) * per_step + k;
    const int nblk = (p.seq_lens[b] + kBlockSize - 1) / kBlockSize;
    if (bi >= nblk) return -1;
    const int32_t blk = p.block_table[(int64_t)b * p.bt_stride + bi];
    if (blk < 0 || blk >= p.num_blocks) {
      report_error(p.err, TQ_DEVERR_BLOCK_RANGE);
      return -1;
    }
    return blk;
  };
  const int64_t nids = (s1 - s0) * per_step;
  for (int64_t i = tid; i < nids && i < p.ids_cap; i += nthreads)
    ids[i] = block_id(s0 + i / per_step, (int)(i % per_step));
  __syncthreads();

  // Stage refill for global step s (issued by one warp): one TMA copy per block of
  // the step, completing on full[stage]; present[stage] tells the consumers which
  // blocks were staged.  With copy_mode 1 the block is a 2-D box of 16 rows whose
  // width is the padded pitch: the columns past the row end lie outside the tensor
  // and are zero-filled, which pads every row in shared memory.
  const uint32_t blk_copy_bytes = p.copy_mode ? (uint32_t)blk_smem : (uint32_t)(kBlockSize * row_bytes);
  auto refill = [&](int64_t s) {
    const int x = (int)((s - s0) % NST);
    const int64_t i0 = (s - s0) * per_step;
    int32_t blk = -1;
    if (lane < per_step) blk = i0 + lane < p.ids_cap ? ids[i0 + lane] : block_id(s, lane);
    const uint32_t bits = __ballot_sync(0xffffffffu, blk >= 0);
    if (lane == 0) {
      present[x] = bits;                 // published by the arrive (release) below
      mbar_arrive_expect_tx(&full[x], __popc(bits) * blk_copy_bytes);
    }
    __syncwarp();
    if (blk >= 0) {
      uint8_t* d = stages + x * p.stage_bytes + lane * blk_smem;
      if (p.copy_mode) tensor_g2s_2d(d, &tmap, 0, blk * kBlockSize, &full[x]);
      else bulk_g2s(d, p.pages + (int64_t)blk * p.blk_stride, blk_copy_bytes, &full[x]);
    }
  };
  if (warp == 0)
    for (int64_t s = s0; s < s1 && s < s0 + NST; ++s) refill(s);

  LK::build(lutK, cents, tid, nthreads);
  if (!one_lut) LV::build(lutV, cents + (1 << KB), tid, nthreads);
  __syncthreads();

  const int kvh = warp % p.h_kv;
  const int sub = warp / p.h_kv;
  const int G = p.group;
  const uint32_t* lk = lutK + lane;
  const uint32_t* lv = lutV + lane;

  // Layout of the score product S^T = K~ . Qhat^T (M = 16 tokens, N = 8 query heads
  // per head group hh, K = coordinates): this thread holds, for m-tile mt (tokens
  // 16mt..16mt+15) and head group hh, sacc[mt][hh][r] = S^T[token 16mt + gid + 8(r>>1)]
  // [head 8hh + 2tig + (r&1)].  Every value it needs for the softmax of its two heads
  // (2tig, 2tig+1) is therefore local, and the O'^T accumulator columns are the same
  // two heads.
  uint32_t qb[C::KSTEPS][NH][2];     // B fragments of Qhat^T: head 8hh + gid
  float qscale[NH][2];               // heads 8hh + 2tig + {0, 1}
  float Mrun[NH][2], lrun[NH][2];
  float acc[NH][C::MT][4];

  // record of (CTA c, sequence b): index c + b (unique, see cta_of)
  auto flush = [&](int b) {
    float* base = p.part + ((int64_t)(blockIdx.x + b) * p.wph + sub) * (int64_t)p.h_q * (D + 2);
#pragma unroll
    for (int hh = 0; hh < NH; ++hh) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float l = lrun[hh][e];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        const int g = 8 * hh + 2 * tig + e;
        if (gid == 0 && g < G) {
          float* rec = base + (int64_t)(kvh * G + g) * (D + 2);
          rec[0] = Mrun[hh][e];
          rec[1] = l;
        }
      }
      static_for<C::MT>([&](auto MI) {
        constexpr int mt = decltype(MI)::value;
        const int c0 = VS::coord(gid, 2 * mt), c1 = VS::coord(gid, 2 * mt + 1);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int g2 = 8 * hh + 2 * tig + (k & 1);
          const int c = (k >> 1) ? c1 : c0;
          if (g2 < G) base[(int64_t)(kvh * G + g2) * (D + 2) + 2 + c] = acc[hh][mt][k];
        }
      });
    }
  };
  auto start = [&](int b) {
#pragma unroll
    for (int hh = 0; hh < NH; ++hh) {
      const int g = 8 * hh + gid;
      const bool have = g < G;
      const int64_t h = (int64_t)b * p.h_q + kvh * G + (have ? g : 0);
      const uint4* src = (const uint4*)(p.qfrag + (h * 4 + tig) * (2 * C::KSTEPS));
#pragma unroll
      for (int v = 0; v < C::KSTEPS / 2; ++v) {
        const uint4 w = have ? src[v] : make_uint4(0u, 0u, 0u, 0u);
        qb[2 * v][hh][0] = w.x; qb[2 * v][hh][1] = w.y;
        qb[2 * v + 1][hh][0] = w.z; qb[2 * v + 1][hh][1] = w.w;
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int ge = 8 * hh + 2 * tig + e;
        qscale[hh][e] = ge < G ? p.qscale[(int64_t)b * p.h_q + kvh * G + ge] : 0.f;
        Mrun[hh][e] = -INFINITY;
        lrun[hh][e] = 0.f;
      }
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[hh][mt][k] = 0.f;
    }
  };

  int cur_b = locate(s0);
  int local = (int)(s0 - prefix[cur_b]);
  int cur_len = p.seq_lens[cur_b];
  start(cur_b);
  for (int64_t s = s0; s < s1; ++s) {
    const int x = (int)((s - s0) % NST);
    if (!mbar_wait(&full[x], (uint32_t)(((s - s0) / NST) & 1), kWaitLimit)) {
      if (lane == 0) report_error(p.err, TQ_DEVERR_TIMEOUT);
      return;
    }
    const int bi = local * per_step + sub;                // this warp's block
    const int valid = ((present[x] >> sub) & 1u) ? min(kBlockSize, cur_len - bi * kBlockSize) : 0;
    if (valid > 0) {
      const uint8_t* base = stages + x * p.stage_bytes + sub * blk_smem + kvh * p.slot_stride;
      // token t (0..15) of this block lives at base + t * pitch

      // ---- S^T = K~ . Qhat^T: one m-tile of 16 tokens ----
      float sacc[NH][4];
#pragma unroll
      for (int hh = 0; hh < NH; ++hh)
#pragma unroll
        for (int k = 0; k < 4; ++k) sacc[hh][k] = 0.f;
      {
        uint32_t kw0[KS::NW], kw1[KS::NW];
        KS::load(kw0, base + gid * pitch, tig);
        KS::load(kw1, base + (gid + 8) * pitch, tig);
        static_for<C::KSTEPS>([&](auto KSI) {
          constexpr int ks = decltype(KSI)::value;
          const uint32_t a0 = LK::pair_field(lk, field<KS::pos(4 * ks), 2 * KB>(kw0));
          const uint32_t a1 = LK::pair_field(lk, field<KS::pos(4 * ks), 2 * KB>(kw1));
          const uint32_t a2 = LK::pair_field(lk, field<KS::pos(4 * ks + 2), 2 * KB>(kw0));
          const uint32_t a3 = LK::pair_field(lk, field<KS::pos(4 * ks + 2), 2 * KB>(kw1));
#pragma unroll
          for (int hh = 0; hh < NH; ++hh)
            mma_16816(sacc[hh], a0, a1, a2, a3, qb[ks][hh][0], qb[ks][hh][1]);
        });
      }
      // this thread's tokens: r = 0, 1  <->  token gid + 8 r
      float nK[2], nV[2], eV[2];
      bool ok[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int t = gid + 8 * r;
        const uint8_t* sl = base + t * pitch;
        nK[r] = *(const float*)(sl + C::KPACK);
        nV[r] = *(const float*)(sl + p.k_region + C::VPACK);
        // floor at 2^-100 keeps 2^(s - M) finite for rows of (near) zero V norm
        eV[r] = fmaxf(log2_ceilish(nV[r]), -100.0f);
        ok[r] = t < valid;
      }
      uint32_t pb[NH][2];   // [head group][b0b1 | b2b3]
#pragma unroll
      for (int hh = 0; hh < NH; ++hh) {
        float sv[2][2];        // [head e][token r]
        float zmax[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          zmax[e] = -INFINITY;
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float a = sacc[hh][2 * r + e];
            sv[e][r] = ok[r] ? a * nK[r] * qscale[hh][e] : -INFINITY;
            zmax[e] = fmaxf(zmax[e], sv[e][r] + eV[r]);
          }
#pragma unroll
          for (int o = 4; o < 32; o <<= 1)
            zmax[e] = fmaxf(zmax[e], __shfl_xor_sync(0xffffffffu, zmax[e], o));
        }
        // lazy reference: raise M only when the tile beats it by more than 2^8
        const bool raise0 = zmax[0] > Mrun[hh][0] + kLazyRescale;
        const bool raise1 = zmax[1] > Mrun[hh][1] + kLazyRescale;
        if (__any_sync(0xffffffffu, raise0 || raise1)) {
          float alpha[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const bool raise = e ? raise1 : raise0;
            const float Mnew = raise ? zmax[e] : Mrun[hh][e];
            alpha[e] = (Mrun[hh][e] == -INFINITY) ? 0.f : exp2f(Mrun[hh][e] - Mnew);
            lrun[hh][e] *= alpha[e];
            Mrun[hh][e] = Mnew;
          }
#pragma unroll
          for (int mt = 0; mt < C::MT; ++mt) {
            acc[hh][mt][0] *= alpha[0]; acc[hh][mt][1] *= alpha[1];
            acc[hh][mt][2] *= alpha[0]; acc[hh][mt][3] *= alpha[1];
          }
        }
        float pv[2][2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float M = Mrun[hh][e];
          float lsum = 0.f;
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float w = ok[r] ? exp2f(sv[e][r] - M) : 0.f;
            lsum += w;
            // masked tokens may hold stale norms (even NaN): their weight is exactly 0
            pv[e][r] = ok[r] ? w * nV[r] : 0.f;
          }
          lrun[hh][e] += lsum;
        }
        // P~ (token, head) pairs in the C layout, transposed to the B layout of P~^T:
        // b0b1 <- tokens 0..7, b2b3 <- tokens 8..15
        pb[hh][0] = movmatrix_trans(pack_half2(pv[0][0], pv[1][0]));
        pb[hh][1] = movmatrix_trans(pack_half2(pv[0][1], pv[1][1]));
      }

      // ---- O'^T += V~^T . P~^T : one k-step of 16 tokens ----
      {
        uint32_t vw[4][VS::NW];   // tokens A, B, C, D = 2tig + {0, 1, 8, 9}
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int t = 2 * tig + (i & 1) + 8 * (i >> 1);
          VS::load(vw[i], base + t * pitch + p.k_region, gid);
        }
        if constexpr (VS::kInterleaved && (VB == 4 || VB == 2)) {
          // transpose the code nibbles (or crumbs) of tokens A/B and C/D into pair
          // indices: lo holds the even codes of a word, hi the odd ones
          constexpr uint32_t M1 = VB == 4 ? 0x0F0F0F0Fu : 0x33333333u;
          static_for<VS::NW>([&](auto JI) {
            constexpr int j = decltype(JI)::value;
            const uint32_t loAB = (vw[0][j] & M1) | ((vw[1][j] << VB) & ~M1);
            const uint32_t hiAB = ((vw[0][j] >> VB) & M1) | (vw[1][j] & ~M1);
            const uint32_t loCD = (vw[2][j] & M1) | ((vw[3][j] << VB) & ~M1);
            const uint32_t hiCD = ((vw[2][j] >> VB) & M1) | (vw[3][j] & ~M1);
            constexpr int PER = VS::PW / 2;            // m-tiles per word
            static_for<PER>([&](auto KI) {
              constexpr int k = decltype(KI)::value;
              constexpr int mt = j * PER + k;
              const uint32_t a0 = LV::pair_field(lv, bits_of<2 * VB * k, 2 * VB>(loAB));
              const uint32_t a1 = LV::pair_field(lv, bits_of<2 * VB * k, 2 * VB>(hiAB));
              const uint32_t a2 = LV::pair_field(lv, bits_of<2 * VB * k, 2 * VB>(loCD));
              const uint32_t a3 = LV::pair_field(lv, bits_of<2 * VB * k, 2 * VB>(hiCD));
#pragma unroll
              for (int hh = 0; hh < NH; ++hh)
                mma_16816(acc[hh][mt], a0, a1, a2, a3, pb[hh][0], pb[hh][1]);
            });
          });
        } else {
          static_for<C::MT>([&](auto MI) {
            constexpr int mt = decltype(MI)::value;
            constexpr int p0 = VS::pos(2 * mt), p1 = VS::pos(2 * mt + 1);
            const uint32_t a0 = LV::pair(lv, field<p0, VB>(vw[0]), field<p0, VB>(vw[1]));
            const uint32_t a1 = LV::pair(lv, field<p1, VB>(vw[0]), field<p1, VB>(vw[1]));
            const uint32_t a2 = LV::pair(lv, field<p0, VB>(vw[2]), field<p0, VB>(vw[3]));
            const uint32_t a3 = LV::pair(lv, field<p1, VB>(vw[2]), field<p1, VB>(vw[3]));
#pragma unroll
            for (int hh = 0; hh < NH; ++hh)
              mma_16816(acc[hh][mt], a0, a1, a2, a3, pb[hh][0], pb[hh][1]);
          });
        }
      }
    }
    // release the stage; the last warp to do so refills it with step s + NST
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      last = atomicAdd(&released[x], 1) == nwarps - 1;
      if (last) released[x] = 0;
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last && s + NST < s1) refill(s + NST);
    // advance the sequence walk; flush the partial at a sequence boundary
    if (s + 1 < s1) {
      ++local;
      int nb = cur_b;
      while (local >= prefix[nb + 1] - prefix[nb]) { ++nb; local = 0; }
      if (nb != cur_b) {
        flush(cur_b);
        cur_b = nb;
        cur_len = p.seq_lens[cur_b];
        start(cur_b);
      }
    }
  }
  flush(cur_b);
}

// Merge the partial records of one (sequence, query head), then o = R^T (O' / l):
// a FWHT of the rotated-domain output, sign flips and the 1/sqrt(D) scale.  The
// records of sequence b come from CTAs cta_of(first step) .. cta_of(last step),
// record index c + b.  Eight warps split the records; each lane owns D/32
// coordinates.
template <int D>
__global__ void __launch_bounds__(256)
merge_kernel(MergeParams p) {
  constexpr int NW = 8, CPL = D / 32;
  __shared__ float buf[D];
  __shared__ float part_o[NW][D];
  __shared__ float part_l[NW];
  __shared__ float red[NW];
  const int h = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t sb = p.prefix[b], eb = p.prefix[b + 1];
  const int64_t S = p.prefix[gridDim.y], Cn = p.nctas;
  const int64_t rstride = (int64_t)p.h_q * (D + 2);
  const float* hbase = p.part + (int64_t)h * (D + 2);
  float o[CPL];
#pragma unroll
  for (int k = 0; k < CPL; ++k) o[k] = 0.f;
  float l = 0.f;
  int n = 0;
  int64_t c_lo = 0;
  const int wshift = __ffs(p.wph) - 1;               // wph is a power of two
  if (eb > sb) {
    c_lo = cta_of(sb, S, Cn);
    n = (int)(cta_of(eb - 1, S, Cn) - c_lo + 1) << wshift;
  }
  // record i -> record offset, or -1 for a CTA whose step range is empty
  auto rec_index = [&](int i) -> int64_t {
    const int64_t c = c_lo + (i >> wshift);
    if (cta_begin(c, S, Cn) >= cta_begin(c + 1, S, Cn)) return -1;
    return (c + b) * p.wph + (i & (p.wph - 1));
  };
  float M = -INFINITY;
  for (int i = tid; i < n; i += 256) {
    const int64_t r = rec_index(i);
    if (r >= 0) M = fmaxf(M, hbase[r * rstride]);
  }
#pragma unroll
  for (int of = 16; of > 0; of >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, of));
  if (lane == 0) red[warp] = M;
  __syncthreads();
  M = red[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) M = fmaxf(M, red[w]);
  if (M != -INFINITY) {
    for (int i = warp; i < n; i += NW) {
      const int64_t r = rec_index(i);
      if (r < 0) continue;
      const float* rec = hbase + r * rstride;
      const float mi = rec[0];
      const float w = mi == -INFINITY ? 0.f : exp2f(mi - M);
      l += w * rec[1];
#pragma unroll
      for (int k = 0; k < CPL; ++k) o[k] += w * rec[2 + lane + 32 * k];
    }
  }
#pragma unroll
  for (int k = 0; k < CPL; ++k) part_o[warp][lane + 32 * k] = o[k];
  if (lane == 0) part_l[warp] = l;
  __syncthreads();
  if (tid < D) {
    float os = 0.f, ls = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) { os += part_o[w][tid]; ls += part_l[w]; }
    buf[tid] = ls > 0.f ? os / ls : 0.f;
  }
  __syncthreads();
  for (int hs = 1; hs < D; hs <<= 1) {
    float v = 0.f;
    if (tid < D) {
      const float mine = buf[tid], other = buf[tid ^ hs];
      v = (tid & hs) ? other - mine : mine + other;
    }
    __syncthreads();
    if (tid < D) buf[tid] = v;
    __syncthreads();
  }
  if (tid < D) {
    float r = buf[tid] * inv_sqrt_dim<D>();
    r = __uint_as_float(__float_as_uint(r) ^ sign_mask_at(p.sign_seed, tid));
    const int64_t off = (int64_t)b * p.o_bstride + (int64_t)h * p.o_hstride + tid;
    if (p.out_dtype == TQ_F32) ((float*)p.out)[off] = r;
    else if (p.out_dtype == TQ_BF16) ((__nv_bfloat16*)p.out)[off] = __float2bfloat16(r);
    else ((__half*)p.out)[off] = __float2half(r);
  }
}

}  // namespace tq
