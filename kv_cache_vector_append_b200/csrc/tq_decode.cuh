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
// so q is rotated once per sequence, and the output is rotated back once.
//
// Kernel layout.  One persistent kernel per call, one CTA per SM.  The (sequence,
// group of wph blocks) steps of the whole batch are laid end to end and CTA c takes
// the contiguous range [c S/C, (c+1) S/C) of the S steps (stream-K style), so ragged
// batches and single long sequences balance alike.  Inside a CTA one warp serves one
// (KV head, sub-stream):
//   * a CTA walks its range as segments, one per sequence; at the start of a segment
//     the CTA rotates that sequence's queries (sign flips, FWHT in registers and
//     shuffles, 1/sqrt(D)) into shared memory as unit fp16 vectors plus
//     |q'| * scale * log2 e, and each warp loads its fragments;
//   * page blocks (16 tokens x all KV heads; one per sub-stream and step) are staged
//     into shared memory by one TMA copy each (a 2-D box of 16 rows one padding wider
//     than a row, the padding zero-filled out of bounds, or a 1-D bulk copy) into a
//     ring of stages guarded by mbarriers; the last warp to release a stage refills
//     it, so no warp waits for the whole CTA; the padded pitch of 20 (mod 32) words
//     makes the per-thread code loads bank-conflict free;
//   * codes become fp16 through shared-memory tables with one 256-byte row per entry
//     (the K table in the first 128 bytes of a row, the V table in the second, lane l
//     at byte 4l), so a warp's lookups always hit 32 different banks; the tables sit at
//     a 64 KiB-aligned shared-window address, so the address of a lookup keyed by a
//     whole byte of codes is one byte permute; tables hold code PAIRS for bits <= 4
//     (entry x | y << bits = (c[x], c[y])), single codes for 8 bits;
//   * S^T = K~ . Qhat^T on mma.sync m16n8k16 (M = 16 tokens, N = 8 query heads of the
//     group, K = D; fp16 operands, fp32 accumulation); s = acc * nK * |q'| * scale * log2 e;
//   * online softmax in base 2 against a running reference M >= max(s + e(nV)),
//     e(x) = log2 x + 1 from the hardware logarithm (an upper bound), raised only when a tile
//     exceeds it by more than 2^8 (lazy rescale), so the fp16 weights
//     P~ = 2^(s - M) nV stay below 2^9 whatever the V norms;
//   * O'^T += V~^T . P~^T on mma.sync (M = coordinates, N = query heads, K = tokens);
//     the fp16 weights go from the C layout of S^T to the B layout of P~^T with one
//     movmatrix transpose per 8 x 8 tile;
//   * at the end of a segment every warp writes its partial (M, l, O') to record
//     ((CTA + sequence) * wph + sub-stream), an index no other (CTA, sequence) pair
//     shares because the ranges are monotone;
//   * end phase: the CTA publishes its records on each covered sequence's counter
//     (release), then takes its share of the merge items (sequence, query head), dealt
//     round-robin over all CTAs: wait (bounded, acquire) until every CTA covering the
//     sequence has published, fold the head's records, divide by l, then o = R^T O'
//     (FWHT, 1/sqrt(D), sign flips).  The launch is cooperative, so the CTAs that wait
//     are co-resident.
// The coordinate order inside each mma tile is free (a permutation applied to both
// operands of a contraction leaves it unchanged); it is chosen so that every thread
// reads whole 32-bit words of codes, and undone when O' is written to its record.
#pragma once

#include "tq_device.cuh"

namespace tq {

constexpr int kBlockSize = 16;        // tokens per page block
constexpr int kMaxStages = 8;         // deepest stage ring
constexpr float kLazyRescale = 8.0f;  // log2 units
constexpr int kLutRow = 256;          // bytes per table entry (K half, V half)

struct DecodeParams {
  const uint8_t* pages;
  int32_t num_blocks;
  int32_t h_kv;
  int32_t slot_stride;          // bytes between heads inside a row
  int32_t row_pitch;            // bytes between rows in shared memory
  int64_t blk_stride;           // bytes between blocks in global memory
  const int32_t* block_table;
  int64_t bt_stride;            // elements between sequences
  int32_t max_blocks;
  const int32_t* seq_lens;
  int32_t batch;
  const void* q;                // [B, H_q, D]
  int64_t q_bstride, q_hstride; // elements
  int32_t q_dtype;
  void* out;                    // [B, H_q, D]
  int64_t o_bstride, o_hstride; // elements
  int32_t out_dtype;
  int32_t h_q;
  int32_t group;                // G = H_q / H_kv
  float scale_log2;             // softmax scale * log2(e)
  uint64_t sign_seed;
  const float* kc;              // K centroids
  const float* vc;              // V centroids
  int32_t k_region;             // bytes of the K region (offset of the V region)
  int32_t wph;                  // warps (sub-streams) per KV head = blocks per step
  int32_t nst;                  // stages in the ring (<= kMaxStages)
  int32_t stage_bytes;
  int32_t ids_cap;              // block ids of its step range a CTA preloads (entries)
  int32_t copy_mode;            // 1: 2-D tensor box per block (rows padded to row_pitch)
                                // 0: 1-D bulk copy per block (row_pitch = row bytes)
  int32_t lut_bytes;            // bytes of the lookup tables
  // Dynamic shared memory layout (byte offsets from its start).  The tables sit at
  // shared-window address lut_win, a multiple of 65536, so that the address of a table
  // entry is (lut_win | e << 8 | column) with no addition; stages 0 .. n_low-1 lie
  // below the tables, the others above them.
  uint32_t lut_win;
  int32_t lut_off;
  int32_t stage_lo_off;
  int32_t stage_hi_off;
  int32_t n_low;
  int32_t misc_off;             // barriers, q', prefix sums, block ids, merge scratch
  int32_t smem_end;             // bytes of dynamic shared memory the layout spans
  float* part;                  // records [(C + B) * wph][H_q][D + 2]
  unsigned int* counters;       // [B] covering CTAs that published, [B] heads finished;
                                // zero between calls (the last user of a counter clears it)
  unsigned int* err;
  uint32_t wait_ms;             // limit of every bounded wait (milliseconds)
  int32_t withhold_cta;         // test hook: this CTA never announces its records (-1: none)
  // Dense rotation R = hi + lo (bf16 bit patterns, [D][D] row-major) in place of the
  // randomized Hadamard transform when rot_hi is not null: q' = R q, o = R^T O' / l.
  const uint16_t* rot_hi;
  const uint16_t* rot_lo;
  // Uncompressed hot window (absent when hot_k is null): hot_k, hot_v [B, W, H_kv, D]
  // with the last dim contiguous (strides in elements); sequence b also attends to its
  // hot tokens 0 .. hot_lens[b]-1, inside the same softmax.
  const void* hot_k;
  const void* hot_v;
  int64_t hot_bstride, hot_tstride, hot_hstride;
  int32_t hot_dtype;
  int32_t hot_cap;              // W
  const int32_t* hot_lens;
  // QJL residual sketch of the keys (decode_kernel MODE 2): K region = [codes | norm |
  // D sign bits | residual norm gamma]; the sketch's signs come from qjl_seed
  int32_t qjl;
  uint64_t qjl_seed;
};

// Bytes per query head of the QJL mode's sketched-query fragments: (b0, b1) half2 pairs
// for every (k-step, tig), padded by 8 bytes so that the 8 heads of a warp's B
// fragments fall in different banks.
__host__ __device__ constexpr int qjl_qz_stride(int d) { return d / 16 * 32 + 8; }

// Arguments of the hot-window partial (a copy of the fields it reads).
struct HotArgs {
  const void* hot_k;
  const void* hot_v;
  int64_t hot_bstride, hot_tstride, hot_hstride;
  int32_t hot_dtype, hot_cap;
  const int32_t* hot_lens;
  const void* q;
  int64_t q_bstride, q_hstride;
  int32_t q_dtype, group;
  float scale_log2;
  unsigned int* err;
};

// Step range of CTA c out of C over S steps: [floor(c S / C), floor((c+1) S / C)).
__host__ __device__ __forceinline__ int64_t cta_begin(int64_t c, int64_t S, int64_t C) {
  return c * S / C;
}
// The CTA whose range holds step x: the largest c with cta_begin(c) <= x.
__host__ __device__ __forceinline__ int64_t cta_of(int64_t x, int64_t S, int64_t C) {
  return ((x + 1) * C - 1) / S;
}
// Whether CTA c has steps.  Every CTA does when S >= C; callers test that first, and
// the divisions stay out of line so that they are not executed (predicated off) on
// that path.
static __device__ __noinline__ bool cta_has_steps(int64_t c, int64_t S, int64_t C) {
  return cta_begin(c, S, C) < cta_begin(c + 1, S, C);
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
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
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

// ---------------------------------------------------------------------------
// Lookup tables.  Entry e of a table is row e (kLutRow bytes) of the table area at
// the start of dynamic shared memory; lane l reads its copy of the K entry at byte
// 4l of the row and its copy of the V entry at byte 128 + 4l.  For BITS <= 4 an entry
// is a code pair: entry (x | y << BITS) = half2(c[x], c[y]); for BITS > 4 it is a
// single code split in two halves: entry x = half2(hi, lo), hi = fp16(c[x]) and
// lo = fp16(c[x] - hi), so that hi + lo carries c[x] to about 2^-22 (the K contraction
// of 8-bit codes uses both).
// ---------------------------------------------------------------------------
__host__ __device__ constexpr int lut_entries(int bits) {
  return bits <= 4 ? 1 << (2 * bits) : 1 << bits;
}

// lut: the first byte of the tables (shared-window address lut_win)
template <int BITS, int HALF>
__device__ __forceinline__ void lut_build(uint8_t* lut, const float* c, int tid, int nt) {
  constexpr int kEntries = lut_entries(BITS);
  for (int i = tid; i < kEntries * 32; i += nt) {
    const int e = i >> 5, l = i & 31;
    uint32_t v;
    if constexpr (BITS <= 4) {
      v = pack_half2(c[e & ((1 << BITS) - 1)], c[e >> BITS]);
    } else {
      const float hi = __half2float(__float2half_rn(c[e]));
      v = pack_half2(hi, c[e] - hi);
    }
    *(uint32_t*)(lut + e * kLutRow + HALF * 128 + 4 * l) = v;
  }
}

// Table of 2-bit V codes taken four at a time (used where the V codes are read
// interleaved): entry q = a | a' << 2 | b << 4 | b' << 6, the codes of two coordinates
// (a, a' of token A; b, b' of token B), holds {half2(c[a], c[b]), half2(c[a'], c[b'])},
// the A-fragment registers of one m-tile's rows g and g + 8.  The V half of row q holds
// 16 copies of the 8-byte entry; lane l reads copy l % 16 (an 8-byte load is served in
// two 16-lane phases, so a warp's lookups never conflict).
__device__ __forceinline__ void lut_build_vquad(uint8_t* lut, const float* c, int tid, int nt) {
  for (int i = tid; i < 256 * 16; i += nt) {
    const int e = i >> 4, cp = i & 15;
    const uint32_t lo = pack_half2(c[e & 3], c[(e >> 4) & 3]);
    const uint32_t hi = pack_half2(c[(e >> 2) & 3], c[e >> 6]);
    *(uint2*)(lut + e * kLutRow + 128 + 8 * cp) = make_uint2(lo, hi);
  }
}

// Shared-window address (e << 8) | off of the entry e held in the field of LEN bits at
// bit POS of the word array; `off` is lut_win | the lane's column (4 lane, + 128 for
// the V table).
template <int POS, int LEN, int NW>
__device__ __forceinline__ uint32_t lut_addr(const uint32_t (&w)[NW], uint32_t off) {
  constexpr int wi = POS >> 5, o = POS & 31;
  constexpr uint32_t m8 = ((1u << LEN) - 1u) << 8;
  if constexpr (o + LEN <= 32) {
    const uint32_t v = w[wi];
    if constexpr (LEN == 8 && o % 8 == 0) {
      // byte 1 <- byte o/8 of v; bytes 0, 2, 3 <- those of off (its byte 1 is 0)
      return __byte_perm(v, off, 0x7604u | ((uint32_t)(o / 8) << 4));
    } else if constexpr (o >= 8) {
      return ((v >> (o - 8)) & m8) | off;
    } else {
      return ((v << (8 - o)) & m8) | off;
    }
  } else {
    const uint32_t f = (w[wi] >> o) | (w[wi + 1] << (32 - o));
    return ((f << 8) & m8) | off;
  }
}
template <int POS, int LEN>
__device__ __forceinline__ uint32_t lut_addr1(uint32_t w, uint32_t off) {
  const uint32_t a[1] = {w};
  return lut_addr<POS, LEN, 1>(a, off);
}
// Table word at shared-window address addr.
__device__ __forceinline__ uint32_t lut_ld(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
// Two table words (an 8-byte entry) at shared-window address addr.
__device__ __forceinline__ uint2 lut_ld2(uint32_t addr) {
  uint2 v;
  asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// half2 (c[x], c[y]) of the codes x, y of one thread's share (consecutive codes at
// bit POS of the word array: one pair field, or two single-code fields).  For BITS > 4
// *rest receives half2 of the low parts (c[x] - hi[x], c[y] - hi[y]).
template <int BITS, int POS, int NW>
__device__ __forceinline__ uint32_t lut_pair(const uint32_t (&w)[NW], uint32_t off,
                                             uint32_t* rest = nullptr) {
  if constexpr (BITS <= 4) {
    return lut_ld(lut_addr<POS, 2 * BITS>(w, off));
  } else {
    const uint32_t ex = lut_ld(lut_addr<POS, BITS>(w, off));
    const uint32_t ey = lut_ld(lut_addr<POS + BITS, BITS>(w, off));
    if (rest) *rest = __byte_perm(ex, ey, 0x7632);   // high halves: the low parts
    return __byte_perm(ex, ey, 0x5410);              // low halves: fp16(c)
  }
}
// half2 (c[x], c[y]) with x the code at bit POS of w0 and y the code at bit POS of w1.
template <int BITS, int POS, int NW>
__device__ __forceinline__ uint32_t lut_pair2(const uint32_t (&w0)[NW], const uint32_t (&w1)[NW],
                                              uint32_t off) {
  if constexpr (BITS <= 4) {
    const uint32_t x = field<POS, BITS>(w0), y = field<POS, BITS>(w1);
    return lut_ld(((x | (y << BITS)) << 8) | off);
  } else {
    const uint32_t ex = lut_ld(lut_addr<POS, BITS>(w0, off));
    const uint32_t ey = lut_ld(lut_addr<POS, BITS>(w1, off));
    return __byte_perm(ex, ey, 0x5410);              // fp16(c[x]), fp16(c[y])
  }
}

// Online fold of `count` partial records into (M, l, o) (one warp; each lane holds E
// values): load(j, m, l, v) fills record j's reference, sum and this lane's values, or
// leaves them empty (m = -inf).  Records are read in batches of NB with all loads of a
// batch in flight together, and folded in with one rescale per batch.
template <int E, class Load>
__device__ __forceinline__ void fold_records(int count, const Load& load, float& M, float& l,
                                             float (&o)[E]) {
  constexpr int NB = E <= 4 ? 8 : 4;
  for (int j0 = 0; j0 < count; j0 += NB) {
    float mj[NB], lj[NB], vj[NB][E];
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      mj[j] = -INFINITY;
      lj[j] = 0.f;
#pragma unroll
      for (int k = 0; k < E; ++k) vj[j][k] = 0.f;
      if (j0 + j < count) load(j0 + j, mj[j], lj[j], vj[j]);
    }
    float mx = M;
#pragma unroll
    for (int j = 0; j < NB; ++j) mx = fmaxf(mx, mj[j]);
    if (mx == -INFINITY) continue;
    const float f = M == -INFINITY ? 0.f : exp2f(M - mx);
    l *= f;
#pragma unroll
    for (int k = 0; k < E; ++k) o[k] *= f;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const float w = mj[j] == -INFINITY ? 0.f : exp2f(mj[j] - mx);
      l = fmaf(w, lj[j], l);
#pragma unroll
      for (int k = 0; k < E; ++k) o[k] = fmaf(w, vj[j][k], o[k]);
    }
    M = mx;
  }
}

// Transpose of an 8x8 matrix of 16-bit values held in mma fragment layout.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
  uint32_t d;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
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
};

// 2^x with the hardware approximation (relative error about 2^-22; results below
// 2^-126 flush to 0, and 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// An upper bound of log2 x within about 1 for x > 0: the hardware base-2 logarithm
// (absolute error far below 1) plus 1; -inf for zero or subnormal x (flushed), NaN for
// NaN.
__device__ __forceinline__ float log2_bound(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y + 1.0f;
}

// In-warp FWHT of D = 32 E values, lane l holding coordinates l E .. l E + E - 1
// (natural order in and out; no scaling).
template <int E>
__device__ __forceinline__ void warp_fwht(float (&x)[E], int lane) {
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
}

// R[r][lane E + i] for i < E (hi + lo, exact in fp32), E = D / 32 consecutive entries.
template <int E>
__device__ __forceinline__ void rot_row_part(const uint16_t* hi, const uint16_t* lo, int r,
                                             int lane, float (&v)[E]) {
  constexpr int D = 32 * E;
  const int64_t o = (int64_t)r * D + lane * E;   // E consecutive entries, 2E-byte aligned
  uint32_t h[E / 2], l[E / 2];
  if constexpr (E == 2) {
    h[0] = *(const uint32_t*)(hi + o);
    l[0] = *(const uint32_t*)(lo + o);
  } else if constexpr (E == 4) {
    const uint2 a = *(const uint2*)(hi + o), b = *(const uint2*)(lo + o);
    h[0] = a.x; h[1] = a.y; l[0] = b.x; l[1] = b.y;
  } else {
    const uint4 a = *(const uint4*)(hi + o), b = *(const uint4*)(lo + o);
    h[0] = a.x; h[1] = a.y; h[2] = a.z; h[3] = a.w;
    l[0] = b.x; l[1] = b.y; l[2] = b.z; l[3] = b.w;
  }
#pragma unroll
  for (int i = 0; i < E / 2; ++i) {
    v[2 * i] = __uint_as_float(h[i] << 16) + __uint_as_float(l[i] << 16);
    v[2 * i + 1] = __uint_as_float(h[i] & 0xffff0000u) + __uint_as_float(l[i] & 0xffff0000u);
  }
}

// sc[0 .. D) <- R sc[0 .. D) for one warp (sc: this warp's shared scratch).  Rounds of
// 16 outputs: every lane loads its E columns of the 16 rows (all loads of a round in
// flight together) and forms its 16 partial dot products; a reduce-scatter over the lane
// bits 3..0 (lane l keeps output l mod 16, 15 shuffles) and one more over bit 4 sum
// them over the warp in fp32.  Out of line, so that it leaves the register allocation of
// the caller's step loop alone.
template <int E>
__device__ __noinline__ void dense_forward(const uint16_t* hi, const uint16_t* lo, float* sc,
                                           int lane) {
  constexpr int D = 32 * E;
  constexpr int CH = 16;
  float x[E];
#pragma unroll
  for (int i = 0; i < E; ++i) x[i] = sc[lane * E + i];
  __syncwarp();
  for (int c0 = 0; c0 < D; c0 += CH) {
    float p[CH];
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      float r[E];
      rot_row_part<E>(hi, lo, c0 + j, lane, r);
      p[j] = 0.f;
#pragma unroll
      for (int i = 0; i < E; ++i) p[j] = fmaf(r[i], x[i], p[j]);
    }
#pragma unroll
    for (int m = CH / 2; m > 0; m >>= 1) {
      const bool up = (lane & m) != 0;      // keep outputs [m, 2m) of the current set
#pragma unroll
      for (int j = 0; j < m; ++j) {
        const float keep = up ? p[j + m] : p[j];
        const float send = up ? p[j] : p[j + m];
        p[j] = keep + __shfl_xor_sync(0xffffffffu, send, m);
      }
    }
    const float out = p[0] + __shfl_xor_sync(0xffffffffu, p[0], 16);
    if (lane < CH) sc[c0 + lane] = out;
  }
  __syncwarp();
}

// sc[0 .. D) <- R^T sc[0 .. D) for one warp: o_c = sum_j R[j][c] a_j in fp32 over
// j = 0 .. D-1 (out of line, as dense_forward).
template <int E>
__device__ __noinline__ void dense_inverse(const uint16_t* hi, const uint16_t* lo, float* sc,
                                           int lane) {
  constexpr int D = 32 * E;
  float a[E];
#pragma unroll
  for (int i = 0; i < E; ++i) a[i] = 0.f;
  __syncwarp();
#pragma unroll 16
  for (int j = 0; j < D; ++j) {
    float r[E];
    rot_row_part<E>(hi, lo, j, lane, r);
    const float aj = sc[j];
#pragma unroll
    for (int i = 0; i < E; ++i) a[i] = fmaf(r[i], aj, a[i]);
  }
  __syncwarp();
#pragma unroll
  for (int i = 0; i < E; ++i) sc[lane * E + i] = a[i];
  __syncwarp();
}

__device__ __forceinline__ float load_as_f32(const void* base, int64_t i, int32_t dtype) {
  if (dtype == TQ_F32) return ((const float*)base)[i];
  if (dtype == TQ_BF16) return __bfloat162float(((const __nv_bfloat16*)base)[i]);
  return __half2float(((const __half*)base)[i]);
}

// Attention partial of query head h of sequence b over its hot-window tokens, computed
// by one warp in the original (unrotated) domain: lane l handles coordinates
// l E .. l E + E - 1.  With s_t = scale log2(e) <q, k_t> (fp32): M = max_t s_t,
// L = sum_t 2^(s_t - M), o = sum_t 2^(s_t - M) v_t, written to sc[0] = M, sc[1] = L,
// sc[2 + c] = o_c (this warp's shared scratch).  A hot_lens entry outside [0, W] raises
// TQ_DEVERR_SEQLEN_RANGE and counts as 0 tokens.  Out of line, as dense_forward.
template <typename T>
__device__ __forceinline__ float as_f32(T x) {
  if constexpr (std::is_same<T, float>::value) return x;
  else return to_f32(x);
}

template <int D, typename T>
__device__ __forceinline__ void hot_partial_t(const HotArgs& a, int b, int h, int lane,
                                              float* sc) {
  constexpr int E = D / 32;
  float M = -INFINITY, L = 0.f, o[E];
#pragma unroll
  for (int i = 0; i < E; ++i) o[i] = 0.f;
  int n = a.hot_lens[b];
  if (n < 0 || n > a.hot_cap) {
    if (lane == 0) report_error(a.err, TQ_DEVERR_SEQLEN_RANGE);
    n = 0;
  }
  float qv[E];
  const int64_t qo = (int64_t)b * a.q_bstride + (int64_t)h * a.q_hstride + lane * E;
#pragma unroll
  for (int i = 0; i < E; ++i) qv[i] = load_as_f32(a.q, qo + i, a.q_dtype);
  const T* hk = (const T*)a.hot_k;
  const T* hv = (const T*)a.hot_v;
  const int64_t base = (int64_t)b * a.hot_bstride + (int64_t)(h / a.group) * a.hot_hstride +
                       lane * E;
  // TPI tokens an iteration, their K and V rows all loaded at its top (one round trip
  // to memory per iteration); independent reductions
  constexpr int TPI = E <= 4 ? 8 : 4;
  for (int t0 = 0; t0 < n; t0 += TPI) {
    float kx[TPI][E], vx[TPI][E];
#pragma unroll
    for (int j = 0; j < TPI; ++j) {
      const bool in = t0 + j < n;
      const int64_t off = base + (int64_t)(in ? t0 + j : 0) * a.hot_tstride;
#pragma unroll
      for (int i = 0; i < E; ++i) {
        kx[j][i] = in ? as_f32(hk[off + i]) : 0.f;
        vx[j][i] = in ? as_f32(hv[off + i]) : 0.f;
      }
    }
    float dot[TPI];
#pragma unroll
    for (int j = 0; j < TPI; ++j) {
      dot[j] = 0.f;
#pragma unroll
      for (int i = 0; i < E; ++i) dot[j] = fmaf(qv[i], kx[j][i], dot[j]);
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1)
#pragma unroll
      for (int j = 0; j < TPI; ++j) dot[j] += __shfl_xor_sync(0xffffffffu, dot[j], m);
    float mx = M;
#pragma unroll
    for (int j = 0; j < TPI; ++j) {
      dot[j] = t0 + j < n ? dot[j] * a.scale_log2 : -INFINITY;
      mx = fmaxf(mx, dot[j]);
    }
    if (mx > M) {
      const float f = M == -INFINITY ? 0.f : exp2f(M - mx);
      L *= f;
#pragma unroll
      for (int i = 0; i < E; ++i) o[i] *= f;
      M = mx;
    }
#pragma unroll
    for (int j = 0; j < TPI; ++j) {
      if (t0 + j < n) {
        const float w = exp2f(dot[j] - M);
        L += w;
#pragma unroll
        for (int i = 0; i < E; ++i) o[i] = fmaf(w, vx[j][i], o[i]);
      }
    }
  }
  __syncwarp();
  if (lane == 0) {
    sc[0] = M;
    sc[1] = L;
  }
#pragma unroll
  for (int i = 0; i < E; ++i) sc[2 + lane * E + i] = o[i];
  __syncwarp();
}

// Attention partial of query head h of sequence b over its hot-window tokens, computed
// by one warp in the original (unrotated) domain: lane l handles coordinates
// l E .. l E + E - 1.  With s_t = scale log2(e) <q, k_t> (fp32): M = max_t s_t,
// L = sum_t 2^(s_t - M), o = sum_t 2^(s_t - M) v_t, written to sc[0] = M, sc[1] = L,
// sc[2 + c] = o_c (this warp's shared scratch).  A hot_lens entry outside [0, W] raises
// TQ_DEVERR_SEQLEN_RANGE and counts as 0 tokens.  Out of line, as dense_forward.
template <int D>
__device__ __noinline__ void hot_partial(const HotArgs a, int b, int h, int lane, float* sc) {
  if (a.hot_dtype == TQ_F32) hot_partial_t<D, float>(a, b, h, lane, sc);
  else if (a.hot_dtype == TQ_BF16) hot_partial_t<D, __nv_bfloat16>(a, b, h, lane, sc);
  else hot_partial_t<D, __half>(a, b, h, lane, sc);
}

__device__ __forceinline__ void store_from_f32(void* base, int64_t i, int32_t dtype, float v) {
  if (dtype == TQ_F32) ((float*)base)[i] = v;
  else if (dtype == TQ_BF16) ((__nv_bfloat16*)base)[i] = __float2bfloat16(v);
  else ((__half*)base)[i] = __float2half(v);
}

// Shared memory: stages below and above the tables (see DecodeParams), and a misc
// area [full mbarriers | release counters | present masks | q' (H_q x D fp16) | |q'|
// scales | step prefix sums | block ids | scan scratch | flag | merge partials |
// record positions].
// MODE 0: the plain kernel.  MODE 1 (EXT): also serves the hot window and the dense
// rotation (runtime choices, both outside the step loop).  MODE 2 (QJL): keys carry the
// QJL sketch of their residual, scored as
//   s = scale nK (<q', c[idx]> + gamma sqrt(pi/2)/sqrt(D) <S q', 2z - 1>)
// with S the sketch's randomized Hadamard transform (a second mma per k-step on +-1
// fragments built from the sign bits).
template <int D, int KB, int VB, int NH, int MAXW, int MODE>
__global__ void __launch_bounds__(MAXW * 32, 1)
decode_kernel(DecodeParams p, const __grid_constant__ CUtensorMap tmap) {
  constexpr bool EXT = MODE == 1;
  constexpr bool QJL = MODE == 2;
  constexpr int QZS = qjl_qz_stride(D);
  using C = DecodeCfg<D, KB, VB>;
  using KS = typename C::KS;
  using VS = typename C::VS;
  constexpr int E = D / 32;
  // 2-bit V codes read interleaved are looked up four at a time (lut_build_vquad)
  constexpr bool VQUAD = VS::kInterleaved && VB == 2;
  extern __shared__ __align__(16) uint8_t smem[];
  {
    // the layout planned on the host must match this launch: tables at lut_win and
    // everything inside the allocation (else report and stop, touching nothing)
    uint32_t dyn_bytes;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_bytes));
    if (smem_u32(smem) + (uint32_t)p.lut_off != p.lut_win || (uint32_t)p.smem_end > dyn_bytes) {
      if (threadIdx.x == 0) report_error(p.err, TQ_DEVERR_LAYOUT);
      return;
    }
  }
  const int nst = p.nst;
  auto stage_ptr = [&](int x) -> uint8_t* {
    return smem + (x < p.n_low ? p.stage_lo_off + x * p.stage_bytes
                               : p.stage_hi_off + (x - p.n_low) * p.stage_bytes);
  };
  uint64_t* full = (uint64_t*)(smem + p.misc_off);
  int* released = (int*)(full + nst);
  uint32_t* present = (uint32_t*)(released + nst);     // per stage: bit k = block k staged
  __half* qh = (__half*)(present + nst);               // unit q' of the current sequence
  float* qsc = (float*)(qh + p.h_q * D);               // |q'| * scale * log2 e
  // QJL: S q' / |q'| of every query head in mma B-fragment order (QZS bytes a head)
  uint8_t* qz = (uint8_t*)(((uintptr_t)(qsc + p.h_q) + 15) & ~(uintptr_t)15);
  int32_t* prefix = (int32_t*)(qz + (QJL ? (p.h_q * QZS + 15) / 16 * 16 : 0));
  int32_t* ids = (int32_t*)(prefix + p.batch + 1);     // block ids of the range
  int* wsum = (int*)(ids + p.ids_cap);                 // [32] per-warp sums of the scan
  int* timed_out = wsum + 32;                          // a stage wait of this CTA gave up
  int* merge_gave_up = timed_out + 1;                  // a merge wait of this CTA gave up
  float* scratch = (float*)(timed_out + 4);            // [warps][D + 2] merge partials
  int* rpos = (int*)(scratch + blockDim.x / 32 * (D + 2));  // [D] coordinate at a record position
  int32_t* lens = (int32_t*)(rpos + D);                // [B] sequence lengths (0 if rejected)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the first copies need the tensor map: fetch it while the prefix sums run
  if (tid == 0 && p.copy_mode)
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap)) : "memory");
  const int gid = lane >> 2, tig = lane & 3;
  auto hot_args = [&]() {
    HotArgs a;
    a.hot_k = p.hot_k;
    a.hot_v = p.hot_v;
    a.hot_bstride = p.hot_bstride;
    a.hot_tstride = p.hot_tstride;
    a.hot_hstride = p.hot_hstride;
    a.hot_dtype = p.hot_dtype;
    a.hot_cap = p.hot_cap;
    a.hot_lens = p.hot_lens;
    a.q = p.q;
    a.q_bstride = p.q_bstride;
    a.q_hstride = p.q_hstride;
    a.q_dtype = p.q_dtype;
    a.group = p.group;
    a.scale_log2 = p.scale_log2;
    a.err = p.err;
    return a;
  };
  const int nthreads = blockDim.x;
  const int nwarps = nthreads >> 5;                    // = h_kv * wph
  const int wph = p.wph;                               // blocks per pipeline step
  const int B = p.batch;


  // ---- step prefix sums over the sequences (every CTA) ----
  {
    const int chunk = (B + nthreads - 1) / nthreads;
    const int lo = tid * chunk, hi = min(B, lo + chunk);
    int sum = 0;
    for (int b = lo; b < hi; ++b) {
      const int len = p.seq_lens[b];
      int steps = 0;
      if (len < 0 || len > p.max_blocks * kBlockSize) {
        if (blockIdx.x == 0) report_error(p.err, TQ_DEVERR_SEQLEN_RANGE);
        lens[b] = 0;
      } else {
        steps = ((len + kBlockSize - 1) / kBlockSize + wph - 1) / wph;
        lens[b] = len;
      }
      prefix[b + 1] = steps;
      sum += steps;
    }
    if (tid < nst) {
      mbar_init(&full[tid], 1);
      released[tid] = 0;
    }
    if (tid == 0) {
      *timed_out = 0;
      *merge_gave_up = 0;
    }
    fence_mbar_init();
    // exclusive scan of the per-thread sums: in each warp, then over the warp totals
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += t;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    if (warp == 0) {
      const int w = lane < nwarps ? wsum[lane] : 0;
      int wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += t;
      }
      if (lane < nwarps) wsum[lane] = wi - w;
      if (lane == 0) prefix[0] = 0;
    }
    __syncthreads();
    int run = wsum[warp] + inc - sum;
    for (int b = lo; b < hi; ++b) { run += prefix[b + 1]; prefix[b + 1] = run; }
    __syncthreads();
  }
  // sequences without steps (empty or rejected) give 0, or attend to their hot window
  // alone (one warp per query head)
  for (int b = blockIdx.x; b < B; b += gridDim.x) {
    if (prefix[b + 1] != prefix[b]) continue;
    if (!EXT || p.hot_k == nullptr) {
      for (int i = tid; i < p.h_q * D; i += nthreads)
        store_from_f32(p.out, (int64_t)b * p.o_bstride + (int64_t)(i / D) * p.o_hstride + i % D,
                       p.out_dtype, 0.f);
    } else {
      float* sc = scratch + warp * (D + 2);
      for (int h = warp; h < p.h_q; h += nwarps) {
        hot_partial<D>(hot_args(), b, h, lane, sc);
        const float L = sc[1];
        const float inv = L > 0.f ? 1.0f / L : 0.f;
        const int64_t ob = (int64_t)b * p.o_bstride + (int64_t)h * p.o_hstride + lane * E;
#pragma unroll
        for (int i = 0; i < E; ++i)
          store_from_f32(p.out, ob + i, p.out_dtype, sc[2 + lane * E + i] * inv);
        __syncwarp();
      }
    }
  }
  const int64_t S = prefix[B];
  const int64_t Cn = gridDim.x;
  const int64_t s0 = cta_begin(blockIdx.x, S, Cn), s1 = cta_begin(blockIdx.x + 1, S, Cn);
  if (s0 >= s1) return;
  // sequence walk: the largest b with prefix[b] <= s
  auto locate = [&](int64_t s) {
    int lo = 0, hi = B;                 // prefix[lo] <= s < prefix[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= s) lo = mid; else hi = mid;
    }
    return lo;
  };

  // the first segment's query heads (the first KPRE of this warp), loaded now so that
  // their latency overlaps the block-id loads and the table build
  const int b_first = locate(s0);
  constexpr int KPRE = 2;
  float qpre[KPRE][E];
#pragma unroll
  for (int k = 0; k < KPRE; ++k) {
    const int h = warp + k * nwarps;
    const int64_t off = (int64_t)b_first * p.q_bstride + (int64_t)(h < p.h_q ? h : 0) * p.q_hstride +
                        lane * E;
#pragma unroll
    for (int i = 0; i < E; ++i) qpre[k][i] = h < p.h_q ? load_as_f32(p.q, off + i, p.q_dtype) : 0.f;
  }

  const int pitch = p.row_pitch;
  const int blk_smem = kBlockSize * pitch;
  const int row_bytes = p.h_kv * p.slot_stride;
  // Block id of block k of global step s: -1 past the end of its sequence or when the
  // table entry is out of range (reported).  The ids of the whole step range are
  // preloaded into shared memory below (up to ids_cap of them) so that a refill never
  // waits on a global load.
  auto block_id = [&](int64_t s, int k) -> int32_t {
    const int b = locate(s);
    const int bi = (int)(s - prefix[b]) * wph + k;
    const int nblk = (lens[b] + kBlockSize - 1) / kBlockSize;
    if (bi >= nblk) return -1;
    const int32_t blk = p.block_table[(int64_t)b * p.bt_stride + bi];
    if (blk < 0 || blk >= p.num_blocks) {
      report_error(p.err, TQ_DEVERR_BLOCK_RANGE);
      return -1;
    }
    return blk;
  };
  // Block ids: warp 0 resolves those of the first nst steps and issues their copies at
  // once (below); the other warps preload the rest of the range meanwhile.
  const int64_t nids = imin64((s1 - s0) * wph, p.ids_cap);
  const int64_t nfirst = imin64((int64_t)nst * wph, nids);
  {
    const int first_t = nwarps > 1 ? 32 : 0;          // a lone warp preloads the rest too
    if (tid >= first_t)
      for (int64_t i = nfirst + tid - first_t; i < nids; i += nthreads - first_t)
        ids[i] = block_id(s0 + i / wph, (int)(i % wph));
  }

  // Stage refill for global step s into stage x (issued by one warp): one TMA copy per
  // block of the step, completing on full[x]; present[x] tells the consumers which
  // blocks were staged.
  const uint32_t blk_copy_bytes =
      p.copy_mode ? (uint32_t)blk_smem : (uint32_t)(kBlockSize * row_bytes);
  auto refill = [&](int64_t s, int x) {
    const int64_t i0 = (s - s0) * wph;
    int32_t blk = -1;
    if (lane < wph) blk = i0 + lane < p.ids_cap ? ids[i0 + lane] : block_id(s, lane);
    const uint32_t bits = __ballot_sync(0xffffffffu, blk >= 0);
    if (lane == 0) {
      present[x] = bits;                 // published by the arrive (release) below
      mbar_arrive_expect_tx(&full[x], __popc(bits) * blk_copy_bytes);
    }
    __syncwarp();
    if (blk >= 0) {
      uint8_t* d = stage_ptr(x) + lane * blk_smem;
      if (p.copy_mode) tensor_g2s_2d(d, &tmap, 0, blk * kBlockSize, &full[x]);
      else bulk_g2s(d, p.pages + (int64_t)blk * p.blk_stride, blk_copy_bytes, &full[x]);
    }
  };
  // The first nst steps: one lane per (stage, block) resolves its block id and issues
  // its copy, all in one pass (a stage's lanes lie in one 32-lane round: wph divides 32).
  if (warp == 0) {
    const int nfs = (int)imin64(nst, s1 - s0);
    const int lwp = __ffs(wph) - 1;
    const uint32_t stage_mask = wph >= 32 ? 0xffffffffu : (1u << wph) - 1u;
    for (int j0 = 0; j0 < nfs * wph; j0 += 32) {
      const int j = j0 + lane;
      const int x = j >> lwp, k = j & (wph - 1);
      const bool in = j < nfs * wph;
      const int32_t blk = in ? block_id(s0 + x, k) : -1;
      const uint32_t bits = __ballot_sync(0xffffffffu, blk >= 0);
      if (in && k == 0) {
        const uint32_t mask = (bits >> lane) & stage_mask;
        present[x] = mask;               // published by the arrive (release) below
        mbar_arrive_expect_tx(&full[x], __popc(mask) * blk_copy_bytes);
      }
      __syncwarp();
      if (blk >= 0) {
        uint8_t* d = stage_ptr(x) + k * blk_smem;
        if (p.copy_mode) tensor_g2s_2d(d, &tmap, 0, blk * kBlockSize, &full[x]);
        else bulk_g2s(d, p.pages + (int64_t)blk * p.blk_stride, blk_copy_bytes, &full[x]);
      }
    }
  }

  // tables (they depend on nothing but the centroids) while the copies and the query
  // loads are in flight
  lut_build<KB, 0>(smem + p.lut_off, p.kc, tid, nthreads);
  if constexpr (VQUAD) lut_build_vquad(smem + p.lut_off, p.vc, tid, nthreads);
  else lut_build<VB, 1>(smem + p.lut_off, p.vc, tid, nthreads);
  // coordinate held at each record position 2 + i (the fragment order; see flush)
  for (int i = tid; i < D; i += nthreads) {
    const int g = i & 7, m = i >> 3;
    rpos[2 * (8 * (m >> 1) + g) + (m & 1)] = VS::coord(g, m);
  }


  const int kvh = warp % p.h_kv;
  const int sub = warp / p.h_kv;
  const int G = p.group;
  const uint32_t lk_off = p.lut_win | (4u * lane);
  const uint32_t lv_off = p.lut_win | (VQUAD ? 128u + 8u * (lane & 15) : 128u + 4u * lane);

  // per warp: q fragments (B operand of the score product), softmax state, O'^T
  uint32_t qb[C::KSTEPS][NH][2];
  float qscale[NH][2];
  float Mrun[NH][2], lrun[NH][2];
  float acc[NH][C::MT][4];

  // Start sequence b (all warps): q' = R q of its query heads into shared memory, the
  // warps splitting the heads (lane l holds coordinates l E .. l E + E - 1: sign flips,
  // FWHT in registers and shuffles, 1/sqrt(D), then normalised to unit fp16), then
  // every warp reads its B fragments and scales and resets its softmax state and O'.
  // Two CTA barriers; called where all warps are between segments.
  auto start = [&](int b, bool pre) {
    __syncthreads();                    // the previous segment's q' is no longer read
    uint32_t sg[E];
#pragma unroll
    for (int i = 0; i < E; ++i) sg[i] = sign_mask_at(p.sign_seed, lane * E + i);
    auto rotate_head = [&](int h, float (&xq)[E]) {
      if (EXT && p.rot_hi != nullptr) {
        float* sc = scratch + warp * (D + 2);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < E; ++i) sc[lane * E + i] = xq[i];
        dense_forward<E>(p.rot_hi, p.rot_lo, sc, lane);
#pragma unroll
        for (int i = 0; i < E; ++i) xq[i] = sc[lane * E + i];
        __syncwarp();
      } else {
#pragma unroll
        for (int i = 0; i < E; ++i) xq[i] = __uint_as_float(__float_as_uint(xq[i]) ^ sg[i]);
        warp_fwht<E>(xq, lane);
#pragma unroll
        for (int i = 0; i < E; ++i) xq[i] *= inv_sqrt_dim<D>();
      }
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < E; ++i) ss = fmaf(xq[i], xq[i], ss);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float nrm = sqrtf(ss);
      const float inv = nrm > 0.f ? 1.0f / nrm : 0.f;
#pragma unroll
      for (int i = 0; i < E; ++i) qh[h * D + lane * E + i] = __float2half_rn(xq[i] * inv);
      if (lane == 0) qsc[h] = nrm * p.scale_log2;
      if constexpr (QJL) {
        // S q'/|q'| = (1/sqrt(D)) H (s2 * q'/|q'|), stored where the B fragments of the
        // sketch product read it: coordinate c = 32 w + i of word w (bit i of the key's
        // sign word w) goes to k-step 8 (w / 4) + (i % 16) / 2, thread w % 4, pair i % 2,
        // half i / 16
        float zq[E];
#pragma unroll
        for (int i = 0; i < E; ++i)
          zq[i] = __uint_as_float(__float_as_uint(xq[i] * inv) ^ sign_mask_at(p.qjl_seed, lane * E + i));
        warp_fwht<E>(zq, lane);
#pragma unroll
        for (int i = 0; i < E; ++i) {
          const int c = lane * E + i, w = c >> 5, bi = c & 31;
          const int ks = 8 * (w >> 2) + ((bi & 15) >> 1);
          const int off = h * QZS + (ks * 4 + (w & 3)) * 8 + (bi & 1) * 4 + (bi >> 4) * 2;
          *(__half*)(qz + off) = __float2half_rn(zq[i] * inv_sqrt_dim<D>());
        }
      }
    };
    auto load_head = [&](int h, float (&xq)[E]) {
      const int64_t off = (int64_t)b * p.q_bstride + (int64_t)h * p.q_hstride + lane * E;
#pragma unroll
      for (int i = 0; i < E; ++i) xq[i] = load_as_f32(p.q, off + i, p.q_dtype);
    };
#pragma unroll
    for (int k = 0; k < KPRE; ++k) {
      const int h = warp + k * nwarps;
      if (h < p.h_q) {
        float xq[E];
        if (pre) {
#pragma unroll
          for (int i = 0; i < E; ++i) xq[i] = qpre[k][i];
        } else {
          load_head(h, xq);
        }
        rotate_head(h, xq);
      }
    }
    for (int h = warp + KPRE * nwarps; h < p.h_q; h += nwarps) {
      float xq[E];
      load_head(h, xq);
      rotate_head(h, xq);
    }
    __syncthreads();
#pragma unroll
    for (int hh = 0; hh < NH; ++hh) {
      const int g = 8 * hh + gid;
      const bool have = g < G;
      const __half* qrow = qh + (kvh * G + (have ? g : 0)) * D;
#pragma unroll
      for (int ks = 0; ks < C::KSTEPS; ++ks) {
        const int c0 = KS::coord(tig, 4 * ks), c2 = KS::coord(tig, 4 * ks + 2);
        qb[ks][hh][0] = have ? *(const uint32_t*)(qrow + c0) : 0u;
        qb[ks][hh][1] = have ? *(const uint32_t*)(qrow + c2) : 0u;
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int ge = 8 * hh + 2 * tig + e;
        qscale[hh][e] = ge < G ? qsc[kvh * G + ge] : 0.f;
        Mrun[hh][e] = -INFINITY;
        lrun[hh][e] = 0.f;
      }
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[hh][mt][k] = 0.f;
    }
  };

  // This warp's partial of sequence b -> its record.  Record of query head h (kRec
  // floats, 16-byte aligned): [O', M, l, 2 unused] with O' in fragment order: coordinate
  // VS::coord(g, 2 mt + c) at 2 (8 mt + g) + c, so that each store (one mt, one head
  // column per thread) writes eight contiguous pairs per head.  Records sit at [h][slot][sub] with slot = CTA + b
  // (unique, as a CTA's sequences follow the previous CTA's), so the records of one
  // (b, h), those of the covering CTAs, are contiguous.
  const int64_t nslots = (int64_t)gridDim.x + B;
  constexpr int64_t kRec = D + 4;                    // floats per record
  auto flush = [&](int b) {
    float* base = p.part + ((int64_t)(blockIdx.x + b) * wph + sub) * kRec;
#pragma unroll
    for (int hh = 0; hh < NH; ++hh) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float l = lrun[hh][e];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        const int g = 8 * hh + 2 * tig + e;
        if (g < G) {
          float* rec = base + (int64_t)(kvh * G + g) * nslots * wph * kRec;
          if (gid == 0) *(float2*)(rec + D) = make_float2(Mrun[hh][e], l);
#pragma unroll
          for (int mt = 0; mt < C::MT; ++mt)
            *(float2*)(rec + 2 * (8 * mt + gid)) =
                make_float2(acc[hh][mt][e], acc[hh][mt][e + 2]);
        }
      }
    }
  };

  const bool every_cta_busy = S >= Cn;
  auto nonempty = [&](int64_t c) { return every_cta_busy || cta_has_steps(c, S, Cn); };
  unsigned int* arrived = p.counters;                // covering CTAs that published b's records
  unsigned int* merged = p.counters + B;             // query heads of b finished
  // (M, l) and this lane's E values of a record (16-byte aligned): values at rec + lane E
  auto load_record = [&](const float* rec, float& m, float& ll, float (&v)[E]) {
    const float2 ml = __ldcg((const float2*)(rec + D));
    m = ml.x;
    ll = ml.y;
    if constexpr (E % 4 == 0) {
#pragma unroll
      for (int k = 0; k < E / 4; ++k) {
        const float4 t = __ldcg((const float4*)(rec + lane * E) + k);
        v[4 * k] = t.x;
        v[4 * k + 1] = t.y;
        v[4 * k + 2] = t.z;
        v[4 * k + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < E / 2; ++k) {
        const float2 t = __ldcg((const float2*)(rec + lane * E) + k);
        v[2 * k] = t.x;
        v[2 * k + 1] = t.y;
      }
    }
  };

  // Wait (lane 0, bounded) until all n covering CTAs have published sequence b's
  // records.  After one wait of this CTA has given up, later ones give up at once.
  auto wait_arrived = [&](int b, int n) -> bool {
    int ok = 1;
    if (lane == 0) {
      if (ld_acquire(&arrived[b]) < (unsigned)n) {
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire(&arrived[b]) < (unsigned)n) {
          if (*(volatile int*)merge_gave_up ||
              globaltimer_ns() - t0 > (uint64_t)p.wait_ms * 1000000ull) {
            report_error(p.err, TQ_DEVERR_TIMEOUT);
            *(volatile int*)merge_gave_up = 1;
            ok = 0;
            break;
          }
          __nanosleep(128);
        }
      }
    }
    __syncwarp();
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
  };

  // Output of query head h of sequence b from its merged partial (Mx, L, a), a in
  // natural coordinate order (lane E + i): o = R^T a / L (the dense rotation, or the
  // FWHT, 1/sqrt(D) and the sign flips), joined with the hot window's partial when
  // there is one.  One warp.
  auto finalize = [&](int b, int h, float Mx, float L, float (&acc_o)[E]) {
    const int64_t ob = (int64_t)b * p.o_bstride + (int64_t)h * p.o_hstride + lane * E;
    uint32_t sg[E];                      // sign flips of this lane's output coordinates
#pragma unroll
    for (int i = 0; i < E; ++i) sg[i] = sign_mask_at(p.sign_seed, lane * E + i);
    auto inverse_rotate = [&](float (&a)[E]) {
      if (EXT && p.rot_hi != nullptr) {
        float* sc = scratch + warp * (D + 2);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < E; ++i) sc[lane * E + i] = a[i];
        dense_inverse<E>(p.rot_hi, p.rot_lo, sc, lane);
#pragma unroll
        for (int i = 0; i < E; ++i) a[i] = sc[lane * E + i];
        __syncwarp();
      } else {
        warp_fwht<E>(a, lane);
#pragma unroll
        for (int i = 0; i < E; ++i)
          a[i] = __uint_as_float(__float_as_uint(a[i] * inv_sqrt_dim<D>()) ^ sg[i]);
      }
    };
    if (!EXT || p.hot_k == nullptr) {
      const float inv = L > 0.f ? 1.0f / L : 0.f;
#pragma unroll
      for (int i = 0; i < E; ++i) acc_o[i] *= inv;
      inverse_rotate(acc_o);
#pragma unroll
      for (int i = 0; i < E; ++i) store_from_f32(p.out, ob + i, p.out_dtype, acc_o[i]);
    } else {
      // R^T O' of the packed tokens (not yet divided by L), then one softmax with the hot
      // window's partial: rescale both to the larger reference and divide by the joint sum
      inverse_rotate(acc_o);
      float* sc = scratch + warp * (D + 2);
      hot_partial<D>(hot_args(), b, h, lane, sc);
      const float Mh = sc[0], Lh = sc[1];
      float oh[E];
#pragma unroll
      for (int i = 0; i < E; ++i) oh[i] = sc[2 + lane * E + i];
      __syncwarp();
      const float Mt = fmaxf(Mx, Mh);
      const float f1 = Mx == -INFINITY ? 0.f : exp2f(Mx - Mt);
      const float f2 = Mh == -INFINITY ? 0.f : exp2f(Mh - Mt);
      const float Lt = f1 * L + f2 * Lh;
      const float inv = Lt > 0.f ? 1.0f / Lt : 0.f;
#pragma unroll
      for (int i = 0; i < E; ++i)
        store_from_f32(p.out, ob + i, p.out_dtype, (f1 * acc_o[i] + f2 * oh[i]) * inv);
    }
  };

  // End phase.  The merge work is dealt out as items (b, h): the R = n_b wph records of
  // query head h of sequence b (n_b covering CTAs); item i = b H_q + h goes to the CTA of
  // rank i mod C' among the C' CTAs with steps, so the merge spreads over the whole grid
  // instead of the CTAs that happen to cover a sequence.  A CTA's items are taken by
  // groups of g warps (g as large as its item count allows); each warp folds its share
  // of the item's records, the group's first warp combines the g partials and writes
  // the head's output.  The last head of b to finish clears b's counters.  `dead`: this
  // CTA gave up a stage wait; its items are counted (so that the counters return to
  // zero) but not merged.
  auto end_phase = [&](bool dead) {
    const int Ce = every_cta_busy ? (int)Cn : (int)S;         // CTAs with steps
    const int my = every_cta_busy ? (int)blockIdx.x : (int)s0;  // rank among them
    const int NI = B * p.h_q;                                   // < 2^31 (host check)
    const int m = my < NI ? (NI - my + Ce - 1) / Ce : 0;
    if (m == 0) return;
    int g = 1;
    while (2 * g * min(m, nwarps) <= nwarps) g *= 2;
    const int groups = nwarps / g, gi = warp / g, mi = warp % g;
    int nat[E];                          // coordinate at record position 2 + lane E + k
#pragma unroll
    for (int k = 0; k < E; ++k) nat[k] = rpos[lane * E + k];
    const int lw = __ffs(wph) - 1;                   // wph is a power of two
    // the CTA of step x: 32-bit arithmetic when (x + 1) C fits
    const bool small = (uint64_t)S * (uint64_t)Cn < (1ull << 32);
    auto cta_of_step = [&](int64_t x) -> int64_t {
      return small ? (int64_t)((uint32_t)((x + 1) * Cn - 1) / (uint32_t)S) : cta_of(x, S, Cn);
    };
    for (int k0 = 0; k0 < m; k0 += groups) {
      const int k = k0 + gi;
      int b = -1, h = 0;
      if (k < m) {
        const int i = my + k * Ce;
        b = i / p.h_q;
        h = i - b * p.h_q;
        if (prefix[b + 1] == prefix[b]) b = -1;        // no steps: output written already
      }
      float M = -INFINITY, l = 0.f, o[E];
#pragma unroll
      for (int i = 0; i < E; ++i) o[i] = 0.f;
      bool ok = false;
      if (b >= 0) {
        const int64_t c_lo = cta_of_step(prefix[b]);
        const int64_t c_hi = cta_of_step(prefix[b + 1] - 1);
        int n = (int)(c_hi - c_lo + 1);
        if (!every_cta_busy) {
          n = 0;
          for (int64_t c = c_lo; c <= c_hi; ++c) n += nonempty(c) ? 1 : 0;
        }
        ok = !dead && wait_arrived(b, n);
        if (ok) {
          const int R = (int)(c_hi - c_lo + 1) << lw;
          const int cnt = R > mi ? (R - mi + g - 1) / g : 0;
          const float* hb = p.part + ((int64_t)h * nslots + c_lo + b) * wph * kRec;
          fold_records<E>(cnt, [&](int j, float& mm, float& ll, float (&v)[E]) {
            const int r = mi + j * g;
            const int64_t c = c_lo + (r >> lw);
            if (nonempty(c)) load_record(hb + (int64_t)r * kRec, mm, ll, v);
          }, M, l, o);
        }
      }
      float* sc = scratch + warp * (D + 2);              // natural coordinate order
      if (lane == 0) { sc[0] = M; sc[1] = l; }
#pragma unroll
      for (int i = 0; i < E; ++i) sc[2 + nat[i]] = o[i];
      __syncthreads();
      if (b >= 0 && mi == 0) {
        float Mx = M, L = l, acc_o[E];
        if (g == 1) {
#pragma unroll
          for (int i = 0; i < E; ++i) acc_o[i] = sc[2 + lane * E + i];
        } else {
          // combine the g partials of the group: lane w < g takes partial w's reference
          // and sum, the rescale factors go round by shuffles
          const float* s0w = scratch + (warp + (lane < g ? lane : 0)) * (D + 2);
          const float mw = lane < g ? s0w[0] : -INFINITY;
          const float lwv = lane < g ? s0w[1] : 0.f;
          Mx = mw;
#pragma unroll
          for (int o2 = 16; o2 > 0; o2 >>= 1) Mx = fmaxf(Mx, __shfl_xor_sync(0xffffffffu, Mx, o2));
          const float fw = (lane < g && mw != -INFINITY) ? exp2f(mw - Mx) : 0.f;
          L = fw * lwv;
#pragma unroll
          for (int o2 = 16; o2 > 0; o2 >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o2);
#pragma unroll
          for (int i = 0; i < E; ++i) acc_o[i] = 0.f;
          for (int w = 0; w < g; ++w) {
            const float f = __shfl_sync(0xffffffffu, fw, w);
            const float* s2 = scratch + (warp + w) * (D + 2) + 2 + lane * E;
#pragma unroll
            for (int i = 0; i < E; ++i) acc_o[i] = fmaf(f, s2[i], acc_o[i]);
          }
          if (Mx == -INFINITY) L = 0.f;
        }
        // count the head first (the counter's round trip overlaps the output); the last
        // head of b clears b's counters, every wait on them being over
        unsigned int done = 0;
        if (lane == 0) done = atomicAdd(&merged[b], 1u);
        if (ok) finalize(b, h, Mx, L, acc_o);
        if (lane == 0 && done == (unsigned)p.h_q - 1) {
          atomicExch(&arrived[b], 0u);
          atomicExch(&merged[b], 0u);
        }
      }
      __syncthreads();
    }
  };

  // Outer loop: the segments (one per sequence) of this CTA's step range; inner loop:
  // the steps of a segment.  Segment set-up and write-out stay out of the step loop.
  int cur_b = b_first;
  int x = 0;
  uint32_t phase = 0;
  bool dead = false;                    // a stage wait of this warp gave up
  // step counters relative to s0 (a range is < 2^31 steps); soff = offset of stage x
  const int nsteps = (int)(s1 - s0);
  const int warp_off = sub * blk_smem + kvh * p.slot_stride;
  int soff = p.n_low > 0 ? p.stage_lo_off : p.stage_hi_off;
  for (int r = 0;;) {
    const int seg_end = (int)(imin64(s1, prefix[cur_b + 1]) - s0);
    // tokens of this warp's block still to come in the sequence
    int rem = lens[cur_b] - ((int)(s0 + r - prefix[cur_b]) * wph + sub) * kBlockSize;
    start(cur_b, cur_b == b_first);
    for (; r < seg_end; ++r, rem -= wph * kBlockSize) {
      if (!dead && !mbar_wait(&full[x], phase, p.wait_ms)) {
        if (lane == 0) {
          report_error(p.err, TQ_DEVERR_TIMEOUT);
          *timed_out = 1;
        }
        dead = true;
      }
      const int valid = (!dead && ((present[x] >> sub) & 1u)) ? min(kBlockSize, rem) : 0;
      if (valid > 0) {
        const uint8_t* base = smem + soff + warp_off;
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
            if constexpr (KB <= 4) {
              const uint32_t a0 = lut_pair<KB, KS::pos(4 * ks)>(kw0, lk_off);
              const uint32_t a1 = lut_pair<KB, KS::pos(4 * ks)>(kw1, lk_off);
              const uint32_t a2 = lut_pair<KB, KS::pos(4 * ks + 2)>(kw0, lk_off);
              const uint32_t a3 = lut_pair<KB, KS::pos(4 * ks + 2)>(kw1, lk_off);
  #pragma unroll
              for (int hh = 0; hh < NH; ++hh)
                mma_16816(sacc[hh], a0, a1, a2, a3, qb[ks][hh][0], qb[ks][hh][1]);
            } else {
              // wide codes: the fp16 centroids, then their low parts (c - fp16(c)), so that
              // the scores carry the fp32 table to about 2^-22
              uint32_t r0, r1, r2, r3;
              const uint32_t a0 = lut_pair<KB, KS::pos(4 * ks)>(kw0, lk_off, &r0);
              const uint32_t a1 = lut_pair<KB, KS::pos(4 * ks)>(kw1, lk_off, &r1);
              const uint32_t a2 = lut_pair<KB, KS::pos(4 * ks + 2)>(kw0, lk_off, &r2);
              const uint32_t a3 = lut_pair<KB, KS::pos(4 * ks + 2)>(kw1, lk_off, &r3);
  #pragma unroll
              for (int hh = 0; hh < NH; ++hh) {
                mma_16816(sacc[hh], a0, a1, a2, a3, qb[ks][hh][0], qb[ks][hh][1]);
                mma_16816(sacc[hh], r0, r1, r2, r3, qb[ks][hh][0], qb[ks][hh][1]);
              }
            }
          });
        }
        // QJL: the sketch product Z~ . (S Qhat)^T on +-1 fragments: bit i of the thread's
        // sign word w gives the low half, bit i + 16 the high half (shifted into the fp16
        // sign bit of +1 / -1)
        float saccz[NH][4];
        float kq[2];
        if constexpr (QJL) {
          constexpr int NWZ = D / 128;               // sign words a thread reads per row
#pragma unroll
          for (int hh = 0; hh < NH; ++hh)
#pragma unroll
            for (int k = 0; k < 4; ++k) saccz[hh][k] = 0.f;
          uint32_t zw0[NWZ], zw1[NWZ];
#pragma unroll
          for (int w = 0; w < NWZ; ++w) {
            zw0[w] = *(const uint32_t*)(base + gid * pitch + C::KPACK + 4 + 4 * (tig + 4 * w));
            zw1[w] = *(const uint32_t*)(base + (gid + 8) * pitch + C::KPACK + 4 + 4 * (tig + 4 * w));
          }
#pragma unroll
          for (int r = 0; r < 2; ++r)
            kq[r] = *(const float*)(base + (gid + 8 * r) * pitch + C::KPACK + 4 + D / 8) *
                    (1.2533141373155003f * inv_sqrt_dim<D>());   // gamma sqrt(pi/2)/sqrt(D)
          static_for<C::KSTEPS>([&](auto KSI) {
            constexpr int ks = decltype(KSI)::value;
            constexpr int w = ks / 8, i = 2 * (ks % 8);
            const uint32_t a0 = ((zw0[w] << (15 - i)) & 0x80008000u) ^ 0xBC00BC00u;
            const uint32_t a1 = ((zw1[w] << (15 - i)) & 0x80008000u) ^ 0xBC00BC00u;
            const uint32_t a2 = ((zw0[w] << (14 - i)) & 0x80008000u) ^ 0xBC00BC00u;
            const uint32_t a3 = ((zw1[w] << (14 - i)) & 0x80008000u) ^ 0xBC00BC00u;
  #pragma unroll
            for (int hh = 0; hh < NH; ++hh) {
              const int g = 8 * hh + gid;
              uint2 bz = make_uint2(0u, 0u);
              if (g < G) bz = *(const uint2*)(qz + (kvh * G + g) * QZS + (ks * 4 + tig) * 8);
              mma_16816(saccz[hh], a0, a1, a2, a3, bz.x, bz.y);
            }
          });
        }
        // this thread's tokens: r = 0, 1  <->  token gid + 8 r
        float nK[2], nV[2], eV[2];
        bool ok[2];
  #pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int t = gid + 8 * r;
          const uint8_t* sl = base + t * pitch;
          ok[r] = t < valid;
          nK[r] = *(const float*)(sl + C::KPACK);
          // masked tokens may hold stale norms (even NaN): their V norm is taken as 0
          nV[r] = ok[r] ? *(const float*)(sl + p.k_region + C::VPACK) : 0.f;
          // floor at 2^-100 keeps 2^(s - M) finite for rows of (near) zero V norm
          eV[r] = fmaxf(log2_bound(nV[r]), -100.0f);
        }
        uint32_t pb[NH][2];   // [head group][b0b1 | b2b3]
  #pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
          float sv[2][2];        // [head e][token r]
          float zloc[2];         // this thread's max of s + e(nV) per head
          bool need = false;
  #pragma unroll
          for (int e = 0; e < 2; ++e) {
            zloc[e] = -INFINITY;
  #pragma unroll
            for (int r = 0; r < 2; ++r) {
              float a = sacc[hh][2 * r + e];
              if constexpr (QJL) a = fmaf(kq[r], saccz[hh][2 * r + e], a);
              sv[e][r] = ok[r] ? a * nK[r] * qscale[hh][e] : -INFINITY;
              zloc[e] = fmaxf(zloc[e], sv[e][r] + eV[r]);
            }
            need |= zloc[e] > Mrun[hh][e] + kLazyRescale;
          }
          // lazy reference: raise M only when the tile beats it by more than 2^8 (the
          // tile maxima over the 16 tokens are only formed when some lane needs them)
          if (__any_sync(0xffffffffu, need)) {
            float zmax[2];
  #pragma unroll
            for (int e = 0; e < 2; ++e) {
              zmax[e] = zloc[e];
  #pragma unroll
              for (int o = 4; o < 32; o <<= 1)
                zmax[e] = fmaxf(zmax[e], __shfl_xor_sync(0xffffffffu, zmax[e], o));
            }
            const bool raise0 = zmax[0] > Mrun[hh][0] + kLazyRescale;
            const bool raise1 = zmax[1] > Mrun[hh][1] + kLazyRescale;
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
              const float w = ex2_approx(sv[e][r] - M);   // exactly 0 for masked tokens
              lsum += w;
              pv[e][r] = w * nV[r];
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
          if constexpr (VQUAD) {
            // regroup the 2-bit codes of tokens A/B and C/D by nibble: byte n of lo
            // holds nibble 2n of the first token's word and of the second's, byte n of hi
            // nibble 2n + 1; nibble k (codes 2k, 2k + 1) is m-tile k of the word, one
            // quad lookup giving its rows g and g + 8
            static_for<VS::NW>([&](auto JI) {
              constexpr int j = decltype(JI)::value;
              const uint32_t loAB = (vw[0][j] & 0x0F0F0F0Fu) | ((vw[1][j] << 4) & 0xF0F0F0F0u);
              const uint32_t hiAB = ((vw[0][j] >> 4) & 0x0F0F0F0Fu) | (vw[1][j] & 0xF0F0F0F0u);
              const uint32_t loCD = (vw[2][j] & 0x0F0F0F0Fu) | ((vw[3][j] << 4) & 0xF0F0F0F0u);
              const uint32_t hiCD = ((vw[2][j] >> 4) & 0x0F0F0F0Fu) | (vw[3][j] & 0xF0F0F0F0u);
              static_for<8>([&](auto KI) {
                constexpr int k = decltype(KI)::value;
                constexpr int mt = j * 8 + k;
                const uint2 ab = lut_ld2(lut_addr1<8 * (k >> 1), 8>((k & 1) ? hiAB : loAB, lv_off));
                const uint2 cd = lut_ld2(lut_addr1<8 * (k >> 1), 8>((k & 1) ? hiCD : loCD, lv_off));
  #pragma unroll
                for (int hh = 0; hh < NH; ++hh)
                  mma_16816(acc[hh][mt], ab.x, ab.y, cd.x, cd.y, pb[hh][0], pb[hh][1]);
              });
            });
          } else if constexpr (VS::kInterleaved && (VB == 4 || VB == 2)) {
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
                const uint32_t a0 = lut_ld(lut_addr1<2 * VB * k, 2 * VB>(loAB, lv_off));
                const uint32_t a1 = lut_ld(lut_addr1<2 * VB * k, 2 * VB>(hiAB, lv_off));
                const uint32_t a2 = lut_ld(lut_addr1<2 * VB * k, 2 * VB>(loCD, lv_off));
                const uint32_t a3 = lut_ld(lut_addr1<2 * VB * k, 2 * VB>(hiCD, lv_off));
  #pragma unroll
                for (int hh = 0; hh < NH; ++hh)
                  mma_16816(acc[hh][mt], a0, a1, a2, a3, pb[hh][0], pb[hh][1]);
              });
            });
          } else {
            static_for<C::MT>([&](auto MI) {
              constexpr int mt = decltype(MI)::value;
              constexpr int p0 = VS::pos(2 * mt), p1 = VS::pos(2 * mt + 1);
              const uint32_t a0 = lut_pair2<VB, p0>(vw[0], vw[1], lv_off);
              const uint32_t a1 = lut_pair2<VB, p1>(vw[0], vw[1], lv_off);
              const uint32_t a2 = lut_pair2<VB, p0>(vw[2], vw[3], lv_off);
              const uint32_t a3 = lut_pair2<VB, p1>(vw[2], vw[3], lv_off);
  #pragma unroll
              for (int hh = 0; hh < NH; ++hh)
                mma_16816(acc[hh][mt], a0, a1, a2, a3, pb[hh][0], pb[hh][1]);
            });
          }
        }
      }
      // release the stage; the last warp to do so refills it with step s + nst
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        last = atomicAdd(&released[x], 1) == nwarps - 1;
        if (last) released[x] = 0;
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last && r + nst < nsteps) refill(s0 + r + nst, x);
      ++x;
      soff = x == p.n_low ? p.stage_hi_off : soff + p.stage_bytes;
      if (x == nst) {
        x = 0;
        phase ^= 1u;
        soff = p.n_low > 0 ? p.stage_lo_off : p.stage_hi_off;
      }
    }
    flush(cur_b);
    if (r >= nsteps) break;
    do ++cur_b; while (prefix[cur_b + 1] == prefix[cur_b]);   // next sequence with steps
  }
  // end phase: publish the records of every sequence of the range, then take this
  // CTA's share of the merge work
  __syncthreads();
  if (tid == 0 && (int)blockIdx.x != p.withhold_cta)
    for (int b = b_first; b <= cur_b; ++b)
      if (prefix[b + 1] > prefix[b]) red_add_release(&arrived[b], 1u);
  const bool dead_cta = *(volatile int*)timed_out != 0;
  if (dead_cta) {
    // copies may still be landing in the stages: give them time (bounded); this CTA's
    // merge items are only counted
    if (tid == 0) {
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 100000000ull) __nanosleep(1000);
    }
    __syncthreads();
  }
  end_phase(dead_cta);
}

}  // namespace tq
