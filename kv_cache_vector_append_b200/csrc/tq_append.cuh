// tq_append.cuh -- quantize-append: rotate, norm, Lloyd-Max encode, bit-pack,
// store into page slots.
//
// Follows TorbuQuant (ginkgoq.github.io/TurboQuant), "TQ4 page tensor" diagram and
// the "Quantize" / "Store" stages; tq-kv (shadowgraph.io), "How It Works" step 3
// (randomized Hadamard transform); turboquant_serve 0.1.2, "Architecture" (update():
// rotate, normalize, Lloyd-Max encode, bit-pack, store uint8).
//
// Work layout.  A row is one (token, KV head) vector of K or of V.  Every lane holds
// 64 consecutive coordinates of a row in 32 registers of fp32 pairs (D/64 lanes per
// row), so the FWHT is six register stages (f32x2 add / sub: two fp32 operations per
// instruction) plus log2(D/64) shuffle stages.  A warp owns a tile of 32*64/D
// consecutive (token, KV head) pairs and does its K rows, then its V rows; lane l
// serves row l % ROWS, part l / ROWS.  A kind's rows of a tile sit in shared memory as
// [part][row][64 elements], the 16-byte chunk c of a part row stored at chunk
// c ^ (row & 7) (the 128-byte swizzle of the tensor-copy unit), so that each 8-lane
// phase of a 16-byte shared load touches 8 different bank groups.  Input rows are
// staged one half-tile ahead: by tensor copies (one box per part: 64 elements x the
// tile's heads x its tokens) when the tile is a box of the input, else by cp.async
// into the same layout.  The tile's full slots are staged in shared memory and stored
// with one bulk copy per token when the page pool holds each token's slots
// back to back with 16-byte alignment, else with lanes running over (slot, word).
//
// Encode.  idx = #{i : b_i < u} over the fp32 boundaries.  For bits <= 4 (and when no
// two boundaries share a bucket) the top 12 bits of u's float encoding (sign,
// exponent, 3 mantissa bits) index a byte table holding 4 k0, k0 = #{b_i < lowest
// float of the bucket}; one compare against b[k0] then gives idx exactly.  Otherwise a
// branch-free binary search over the boundaries in Eytzinger order.
#pragma once

#include "tq_device.cuh"

namespace tq {

struct AppendParams {
  uint8_t* pages;
  int64_t num_slots;      // num_blocks * block_size
  int32_t block_size;
  int32_t h_kv;
  int64_t blk_stride;     // bytes
  int64_t row_stride;     // bytes
  int64_t head_stride;    // bytes
  const int64_t* slot_mapping;
  int64_t slot_map_stride;  // elements
  int64_t num_tokens;
  const void* src[2];       // K, V
  int64_t tok_stride[2];    // elements
  int64_t head_stride_in[2];
  const float* boundaries[2];
  int32_t bits[2];
  int32_t region_off[2];    // byte offset of the K / V region inside a slot
  uint64_t sign_seed;
  unsigned int* err;
  int32_t align_mode;       // 16: rows 16-byte aligned; 4: 4-byte aligned; 0: any
  int32_t bs_shift;         // log2(block_size) when it is a power of two, else -1
  int32_t run_heads;        // heads of one token in a tile (tiles token-aligned), else 0
  int32_t tma_in;           // 1: input rows staged by tensor copies (maps K, V)
  int32_t bulk_out;         // 1: slots stored by one bulk copy per token run
  int32_t slot_body;        // > 0 (padded slot stride): slots stored one by one, the first
                            // slot_body bytes (a multiple of 16) by a bulk copy, the rest
                            // by 4-byte stores
  unsigned int* redo;       // [2]: a row left the fast path's range; CTAs of the redo done
  // QJL residual sketch of the keys (append_kernel<..., QJL = true>): K centroids and the
  // seed of the sketch's signs
  const float* kcent;
  uint64_t qjl_seed;
};

// Tensor maps of K and V as (D, h_kv, tokens) 16-bit elements, boxes of
// (64, run_heads, ROWS / run_heads) with the 128-byte swizzle; unused unless tma_in.
struct AppendMaps {
  CUtensorMap k, v;
};

struct RotateParams {      // test export of the rotation (tq_rotate_unit)
  const void* x;
  int64_t x_row_stride;    // elements
  int64_t rows;
  float* u;
  int64_t u_row_stride;
  float* norm;
  int64_t norm_stride;
  uint64_t sign_seed;
  int32_t align_mode;
};

constexpr int kAppendWarps = 8;
constexpr int kBucketShift = 20;                 // 12-bit buckets: sign, exponent, 3 bits
constexpr int kBuckets = 1 << (32 - kBucketShift);

template <int D>
struct AppendGeom {
  static constexpr int E = 64;                        // elements per lane
  static constexpr int TPR = D / E;                   // lanes per row
  static constexpr int ROWS = 32 / TPR;               // rows per warp tile
};

// Shared tables of one kind (K or V), 6 KiB.  The bucket of u is the top 12 bits of
// its float encoding (sign, exponent, 3 mantissa bits); its byte holds 4 k0, where
// k0 = #{b_i < lowest float of the bucket}.  The boundaries start 64-byte aligned, so
// b[k0] sits at shared-window address (bnd address | 4 k0) for bits <= 4; one compare
// against it then gives idx exactly.  Every 12-bit bucket has an entry.
struct alignas(64) EncodeTables {
  uint8_t k4[kBuckets];     // 4 * k0 per bucket
  float bnd[257];           // boundaries b_0..b_{L-2}, then +inf (64-byte aligned)
  float eytz[255];          // Eytzinger image, node e at eytz[e - 1]
};
static_assert(sizeof(EncodeTables) == 6144, "table layout");

// Phase 1 (then a CTA barrier, then phase 2): boundaries and Eytzinger image; thread 0
// records whether the bucket encode applies (no two boundaries share a bucket, and
// the boundaries are 64-byte aligned).
__device__ __forceinline__ void build_tables(EncodeTables* t, const float* b, int bits, int tid,
                                             int nthreads, int* fast) {
  const int n = (1 << bits) - 1;
  for (int i = tid; i <= n; i += nthreads) t->bnd[i] = i < n ? b[i] : INFINITY;
  for (int i = 1 + tid; i <= n; i += nthreads) {
    const int d = 31 - __clz(i);
    const int k = i - (1 << d);
    t->eytz[i - 1] = b[((2 * k + 1) << (bits - 1 - d)) - 1];
  }
  if (tid == 0) {
    int ok = bits <= 4 && (smem_u32(t->bnd) & 63u) == 0;
    for (int i = 0; i + 1 < n; ++i)
      if ((__float_as_uint(b[i]) >> kBucketShift) == (__float_as_uint(b[i + 1]) >> kBucketShift))
        ok = 0;
    *fast = ok;
  }
}

// Phase 2: 4 k0 of each bucket (binary search over the boundaries already in shared
// memory).  The lowest float of bucket g is g << 20 for a positive bucket and
// -((g & 0x7ff) << 20 | 0xfffff) for a negative one.  Only used for bits <= 4.
// Coordinates of a unit vector have |u| <= 1 (up to rounding), so only the buckets of
// |u| < 2 are searched; the others hold their exact counts directly: every boundary
// (|b| < 1) lies below u >= 2, none below u <= -2, and NaN patterns get a valid entry.
__device__ __forceinline__ void build_bucket_table(EncodeTables* t, int bits, int tid,
                                                   int nthreads) {
  if (bits > 4) return;
  const int n = (1 << bits) - 1;
  for (int g = tid; g < kBuckets; g += nthreads) {
    int a;
    if ((g & 0x7ff) >= 0x400) {         // |u| >= 2 (or inf / NaN patterns)
      a = (g & 0x800) ? 0 : n;
    } else {
      const uint32_t lowbits = (g & 0x800) ? ((uint32_t)g << kBucketShift) | 0xFFFFFu
                                           : (uint32_t)g << kBucketShift;
      const float lo = __uint_as_float(lowbits);
      a = 0;
      int c = n;                        // count of boundaries < lo lies in [a, c]
      while (a < c) {
        const int m = (a + c) >> 1;
        if (t->bnd[m] < lo) a = m + 1; else c = m;
      }
    }
    t->k4[g] = (uint8_t)(4 * a);
  }
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

// Stage `nrows` rows of RB bytes into the tile layout [part][row][PB] (16-byte chunk c of
// a part row stored at chunk c ^ (row & 7)); row r starts at row_ptr(r).  Issued by one
// warp.
template <int RB, int PB, int ROWS>
__device__ __forceinline__ uint8_t* tile_at(uint8_t* dst, int r, int b) {
  return dst + (b / PB) * (ROWS * PB) + r * PB + ((((b % PB) >> 4) ^ (r & 7)) << 4) + (b & 15);
}
template <int RB, int PB, int ROWS, typename RowPtr>
__device__ __forceinline__ void stage_rows(uint8_t* dst, int nrows, RowPtr row_ptr,
                                           int align_mode, int lane) {
  if (align_mode == 16) {
    constexpr int NC = RB / 16;
    for (int f = lane; f < nrows * NC; f += 32) {
      const int r = f / NC, b = (f % NC) * 16;
      cp_async16(tile_at<RB, PB, ROWS>(dst, r, b), (const uint8_t*)row_ptr(r) + b);
    }
  } else if (align_mode == 4) {
    constexpr int NC = RB / 4;
    for (int f = lane; f < nrows * NC; f += 32) {
      const int r = f / NC, b = (f % NC) * 4;
      cp_async4(tile_at<RB, PB, ROWS>(dst, r, b), (const uint8_t*)row_ptr(r) + b);
    }
  } else {
    constexpr int NC = RB / 2;
    for (int f = lane; f < nrows * NC; f += 32) {
      const int r = f / NC, b = (f % NC) * 2;
      *(uint16_t*)tile_at<RB, PB, ROWS>(dst, r, b) = *(const uint16_t*)((const uint8_t*)row_ptr(r) + b);
    }
  }
}

// ---------------------------------------------------------------------------
// Packed fp32 pairs.  A lane's 64 coordinates live in 32 64-bit registers, element
// 2i in the low half of register i and 2i+1 in the high half; the add / sub / fma /
// mul of two registers is one f32x2 instruction (two independent IEEE fp32
// operations, each rounded to nearest even, so the results equal those of the
// scalar operations).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float f2lo(uint64_t v) {
  return __uint_as_float((uint32_t)v);
}
__device__ __forceinline__ float f2hi(uint64_t v) {
  return __uint_as_float((uint32_t)(v >> 32));
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// Load this lane's 64 input elements from shared memory as fp32 pairs with the
// rotation signs applied (the sign flip is an xor of the sign bit; for bf16 it rides
// along with the widening), and do the first FWHT stage (h = 1, the two halves of a
// register): (a, b) -> (a + b, a - b).
// `row` is the shared-window address of this lane's part row (aligned to its size) with
// the row's swizzle (row & 7) in bits 4-6, so chunk c sits at row ^ (c << 4).
template <typename Tin>
__device__ __forceinline__ void load_signed(uint64_t (&xp)[32], uint32_t row,
                                            const uint32_t* m) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float a[8];
    const uint4 s0 = *(const uint4*)(m + 8 * c);
    const uint4 s1 = *(const uint4*)(m + 8 * c + 4);
    const uint32_t s[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    if constexpr (sizeof(Tin) == 4) {
      const uint4 q0 = lds128(row ^ (uint32_t)(32 * c));
      const uint4 q1 = lds128(row ^ (uint32_t)(32 * c + 16));
      const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
      for (int k = 0; k < 8; ++k) a[k] = __uint_as_float(w[k] ^ s[k]);
    } else {
      const uint4 q = lds128(row ^ (uint32_t)(16 * c));
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if constexpr (std::is_same<Tin, __nv_bfloat16>::value) {
          a[2 * k + 0] = __uint_as_float((w[k] << 16) ^ s[2 * k]);
          a[2 * k + 1] = __uint_as_float((w[k] & 0xFFFF0000u) ^ s[2 * k + 1]);
        } else {
          __half2 h = *reinterpret_cast<const __half2*>(&w[k]);
          const float2 f = __half22float2(h);
          a[2 * k + 0] = __uint_as_float(__float_as_uint(f.x) ^ s[2 * k]);
          a[2 * k + 1] = __uint_as_float(__float_as_uint(f.y) ^ s[2 * k + 1]);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
      xp[4 * c + k] = f2(__fadd_rn(a[2 * k], a[2 * k + 1]), __fsub_rn(a[2 * k], a[2 * k + 1]));
  }
}

// 2^k as a float, for -126 <= k <= 127.
__device__ __forceinline__ float pow2f(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }

// floor(log2 x) of the positive finite float with bit pattern b (normal or subnormal).
__device__ __forceinline__ int exponent_of(uint32_t b) {
  return b >= 0x00800000u ? (int)(b >> 23) - 127 : (31 - __clz((int)b)) - 149;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint32_t scale_bits(uint32_t w, float s1, float s2) {
  return __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(w), s1), s2));
}

// Rare path of rotate_row.  Every lane of the warp takes part (the row maximum is
// combined over the row's lanes).  For a row with `need` set that holds only finite
// values, not all zero: e = floor(log2 max|x|), and this lane's 64 staged elements are
// multiplied in place by 2^-e (two power-of-two factors, both normal floats; the
// product is exact unless it leaves the normal range, and the 16-bit formats share
// fp32's exponent range for bf16, while f16 rows never need it); returns e, else 0.
// *bad = the row holds an infinity or NaN.
template <int D, typename Tin>
__device__ __noinline__ int rescale_staged_row(uint32_t row, bool need, bool* bad) {
  using G = AppendGeom<D>;
  constexpr int NCH = 64 * (int)sizeof(Tin) / 16;   // 16-byte chunks of the part row
  uint32_t mx = 0u;                                  // |x| as fp32 bits (integer order)
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const uint4 q = lds128(row ^ (uint32_t)(16 * c));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if constexpr (sizeof(Tin) == 4) {
        mx = max(mx, w[k] & 0x7fffffffu);
      } else if constexpr (std::is_same<Tin, __nv_bfloat16>::value) {
        mx = max(mx, (w[k] << 16) & 0x7fffffffu);
        mx = max(mx, w[k] & 0x7fff0000u);
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
        mx = max(mx, __float_as_uint(f.x) & 0x7fffffffu);
        mx = max(mx, __float_as_uint(f.y) & 0x7fffffffu);
      }
    }
  }
#pragma unroll
  for (int m = 1; m < G::TPR; m <<= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, G::ROWS * m));
  *bad = mx >= 0x7f800000u;
  if (!need || *bad || mx == 0u) return 0;
  const int e = exponent_of(mx);
  const float s1 = pow2f(-e / 2), s2 = pow2f(-e - (-e / 2));
#pragma unroll 1
  for (int c = 0; c < NCH; ++c) {
    const uint32_t a = row ^ (uint32_t)(16 * c);
    const uint4 q = lds128(a);
    uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if constexpr (sizeof(Tin) == 4) {
        w[k] = scale_bits(w[k], s1, s2);
      } else if constexpr (std::is_same<Tin, __nv_bfloat16>::value) {
        const uint32_t lo = scale_bits(w[k] << 16, s1, s2) >> 16;   // exact: low bits are 0
        const uint32_t hi = scale_bits(w[k] & 0xffff0000u, s1, s2) & 0xffff0000u;
        w[k] = hi | lo;
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
        const __half2 h = __floats2half2_rn(__fmul_rn(__fmul_rn(f.x, s1), s2),
                                            __fmul_rn(__fmul_rn(f.y, s1), s2));
        w[k] = *reinterpret_cast<const uint32_t*>(&h);
      }
    }
    sts128(a, make_uint4(w[0], w[1], w[2], w[3]));
  }
  // these generic-proxy writes come before any later tensor copy into the buffer
  fence_proxy_async_smem();
  return e;
}

// FWHT stages h = 2, 4, ..., 32 in registers and h = 64, 128 across the lanes of the row
// (stage h = 1 is done by load_signed), then the row's sum of squares of the transformed
// coordinates: even and odd coordinates accumulated separately by fused multiply-add in
// register order, added, then the lanes of a row add their sums pairwise (xor butterfly
// over the part bits), so every lane of the row holds the same value.
template <int D>
__device__ __forceinline__ float fwht_ss(uint64_t (&xp)[32], int part) {
  using G = AppendGeom<D>;
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {           // element stride 2h
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((i & h) == 0) {
        const uint64_t a = xp[i], b = xp[i + h];
        xp[i] = add2(a, b);
        xp[i + h] = sub2(a, b);
      }
    }
  }
#pragma unroll
  for (int m = 1; m < G::TPR; m <<= 1) {
    const float sg = (part & m) ? -1.0f : 1.0f;
    const uint64_t sg2 = f2(sg, sg);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float olo = __shfl_xor_sync(0xffffffffu, f2lo(xp[i]), G::ROWS * m);
      const float ohi = __shfl_xor_sync(0xffffffffu, f2hi(xp[i]), G::ROWS * m);
      // part bit set: o - x; clear: x + o
      xp[i] = fma2(xp[i], sg2, f2(olo, ohi));
    }
  }
  uint64_t ss2 = 0ull;
#pragma unroll
  for (int i = 0; i < 32; ++i) ss2 = fma2(xp[i], xp[i], ss2);
  float ss = __fadd_rn(f2lo(ss2), f2hi(ss2));
#pragma unroll
  for (int m = 1; m < G::TPR; m <<= 1)
    ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, G::ROWS * m));
  return ss;
}

// The rotation shared by quantize-append and its test export.  Loads this lane's 64
// input elements of the row from the staged tile (`row`, `m`: see load_signed) and
// leaves in xp the unnormalised transform H (s * x') of those coordinates, where x' is
// the row scaled by 2^-e; returns r with u = xp * r.  *norm_out = ||x||_2 in fp32.
// The fast path (SAFE = false) takes e = 0 and sets *out_of_range when the sum of
// squares ss of the transform (= D ||x||^2) falls outside [2^-60, 2^100] (squares that
// overflow fp32 or lose precision as subnormals, a zero row, a non-finite row); such a
// call is then redone by the safe path.  The safe path (SAFE = true; also the test
// export) rescales the warp's rows that are out of range in place in the staged tile
// by 2^-e, e = floor(log2 max|x|) (largest magnitude in [1, 2)), and transforms every
// row of the warp again; multiplying by a power of two is exact, so a row in range
// comes out bit for bit as in the fast path.  *bad_out = the row holds an infinity or
// NaN (safe path only).  Order of operations (fixed, so that the export reproduces the
// kernel exactly): the FWHT and ss of fwht_ss; n' = sqrt(ss / D) (IEEE);
// r = 1 / (n' sqrt(D)) (IEEE reciprocal), or 0 when n' == 0; norm = n' 2^e.
template <int D, typename Tin, bool SAFE>
__device__ __forceinline__ float rotate_row(uint64_t (&xp)[32], uint32_t row, const uint32_t* m,
                                            int part, float* norm_out, bool* bad_out,
                                            bool* out_of_range) {
  int e = 0;
  bool bad = false;
  load_signed<Tin>(xp, row, m);
  float ss = fwht_ss<D>(xp, part);
  const bool in_range = ss >= 0x1p-60f && ss <= 0x1p100f;
  if constexpr (SAFE) {
    if (__any_sync(0xffffffffu, !in_range)) {
      e = rescale_staged_row<D, Tin>(row, !in_range, &bad);
      __syncwarp();
      load_signed<Tin>(xp, row, m);
      ss = fwht_ss<D>(xp, part);
    }
  } else {
    *out_of_range = !in_range;
  }
  // ||H s x'||^2 = D ||x'||^2
  const float n = sqrtf(__fmul_rn(ss, 1.0f / D));
  *norm_out = e == 0 ? n : __fmul_rn(__fmul_rn(n, pow2f(e / 2)), pow2f(e - e / 2));
  *bad_out = bad;
  const float sqrt_d = D == 64 ? 8.0f : (D == 128 ? 11.313708498984761f : 16.0f);
  return n > 0.f ? __frcp_rn(__fmul_rn(n, sqrt_d)) : 0.f;
}

// Encode u = x * r and pack the 64 codes LSB-first into 2*BITS words.  RES: also leave
// the residuals u - c[code] in xp (fp32 pairs), with `cent_win` the shared-window address
// of the centroid table.
template <int BITS, bool FAST, bool RES = false>
__device__ __forceinline__ void encode_pack(uint64_t (&xp)[32], float r, const EncodeTables* t,
                                            uint32_t* words, uint32_t cent_win = 0) {
  constexpr int W = 64 * BITS / 32;
  uint32_t acc[W];
#pragma unroll
  for (int w = 0; w < W; ++w) acc[w] = 0u;
  const uint64_t r2 = f2(r, r);
  const uint32_t bnd_win = smem_u32(t->bnd);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint64_t u2 = mul2(xp[i], r2);
    float cv[2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const float u = hf ? f2hi(u2) : f2lo(u2);
      const int j = 2 * i + hf;
      const int bit = j * BITS;
      const int w0 = bit >> 5, o0 = bit & 31;
      // the fields of a word do not overlap, so a shifted add packs the code
      if constexpr (FAST) {
        const uint32_t k4 = t->k4[__float_as_uint(u) >> kBucketShift];
        const uint32_t c4 = k4 + (u > lds_f32(bnd_win | k4) ? 4u : 0u);   // 4 * code
        if (o0 >= 2) acc[w0] += c4 << (o0 - 2);
        else acc[w0] += c4 >> (2 - o0);
        if (o0 + BITS > 32) acc[w0 + 1] += c4 >> (32 - o0 + 2);
        if constexpr (RES) cv[hf] = lds_f32(cent_win + c4);
      } else {
        int e = 1;
#pragma unroll
        for (int st = 0; st < BITS; ++st) e = 2 * e + (u > t->eytz[e - 1] ? 1 : 0);
        const uint32_t code = (uint32_t)(e - (1 << BITS));
        acc[w0] += code << o0;
        if (o0 + BITS > 32) acc[w0 + 1] += code >> (32 - o0);
        if constexpr (RES) cv[hf] = lds_f32(cent_win + 4 * code);
      }
    }
    if constexpr (RES) xp[i] = sub2(u2, f2(cv[0], cv[1]));
  }
#pragma unroll
  for (int w = 0; w < W; ++w) words[w] = acc[w];
}

template <int BITS, bool RES = false>
__device__ __forceinline__ void encode_pack_any(uint64_t (&xp)[32], float r,
                                                const EncodeTables* t, int fast,
                                                uint32_t* words, uint32_t cent_win = 0) {
  if constexpr (BITS <= 4) {
    if (fast) {
      encode_pack<BITS, true, RES>(xp, r, t, words, cent_win);
      return;
    }
  }
  encode_pack<BITS, false, RES>(xp, r, t, words, cent_win);
}

template <bool RES>
__device__ __forceinline__ void encode_pack_bits(int bits, uint64_t (&xp)[32], float r,
                                                 const EncodeTables* t, int fast,
                                                 uint32_t* words, uint32_t cent_win) {
  switch (bits) {
    case 1: encode_pack_any<1, RES>(xp, r, t, fast, words, cent_win); break;
    case 2: encode_pack_any<2, RES>(xp, r, t, fast, words, cent_win); break;
    case 3: encode_pack_any<3, RES>(xp, r, t, fast, words, cent_win); break;
    case 4: encode_pack_any<4, RES>(xp, r, t, fast, words, cent_win); break;
    case 5: encode_pack_any<5, RES>(xp, r, t, fast, words, cent_win); break;
    case 6: encode_pack_any<6, RES>(xp, r, t, fast, words, cent_win); break;
    case 7: encode_pack_any<7, RES>(xp, r, t, fast, words, cent_win); break;
    default: encode_pack_any<8, RES>(xp, r, t, fast, words, cent_win); break;
  }
}

// QJL sketch of this lane's 64 residuals r (in xp): the sketch's sign flips (`qm`, as in
// load_signed), the FWHT (stage h = 1 here, then fwht_ss), and the sign bits
// z_j = [ (S r)_j >= 0 ] of the lane's coordinates into two words (bit j of the lane's
// 64).  Returns gamma = ||r||_2 of the row (the lanes of the row combined).
template <int D>
__device__ __forceinline__ float qjl_sketch_row(uint64_t (&xp)[32], const uint32_t* qm, int part,
                                                uint32_t* z0, uint32_t* z1) {
  using G = AppendGeom<D>;
  uint64_t g2 = 0ull;
#pragma unroll
  for (int i = 0; i < 32; ++i) g2 = fma2(xp[i], xp[i], g2);
  float gg = __fadd_rn(f2lo(g2), f2hi(g2));
#pragma unroll
  for (int m = 1; m < G::TPR; m <<= 1)
    gg = __fadd_rn(gg, __shfl_xor_sync(0xffffffffu, gg, G::ROWS * m));
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 s0 = *(const uint4*)(qm + 8 * c);
    const uint4 s1 = *(const uint4*)(qm + 8 * c + 4);
    const uint32_t sm[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a = __uint_as_float(__float_as_uint(f2lo(xp[4 * c + k])) ^ sm[2 * k]);
      const float b = __uint_as_float(__float_as_uint(f2hi(xp[4 * c + k])) ^ sm[2 * k + 1]);
      xp[4 * c + k] = f2(__fadd_rn(a, b), __fsub_rn(a, b));
    }
  }
  (void)fwht_ss<D>(xp, part);
  uint32_t w0 = 0u, w1 = 0u;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    w0 |= (f2lo(xp[i]) >= 0.f ? 1u : 0u) << (2 * i);
    w0 |= (f2hi(xp[i]) >= 0.f ? 1u : 0u) << (2 * i + 1);
    w1 |= (f2lo(xp[16 + i]) >= 0.f ? 1u : 0u) << (2 * i);
    w1 |= (f2hi(xp[16 + i]) >= 0.f ? 1u : 0u) << (2 * i + 1);
  }
  *z0 = w0;
  *z1 = w1;
  return sqrtf(gg);
}

// Shared memory: the K and V tables and sign masks; then (1024-byte aligned, as the
// swizzled tensor copies need) each warp's two input buffers (K rows, V rows of one
// tile, KIND bytes each); then each warp's small arrays: two mbarriers, the slot
// offsets and row addresses of two tiles, and the tile's slots ([ROWS][slot words]).
template <int D, typename Tin>
struct AppendSmem {
  using G = AppendGeom<D>;
  static constexpr int RB = D * InType<Tin>::kBytes;    // bytes of one input row
  static constexpr int PB = 64 * InType<Tin>::kBytes;   // bytes of one lane's part of a row
  static constexpr int KIND = G::TPR * G::ROWS * PB;    // one kind's rows of a tile
  // K and V tables, sign masks, flags[4], K centroids[256], QJL sign masks
  static constexpr int TABLES =
      ((2 * (int)sizeof(EncodeTables) + 4 * D + 16 + 1024 + 4 * D) + 127) / 128 * 128;
  static __host__ __device__ constexpr int slot_words(int kbits, int vbits) {
    return (D * kbits / 8 + 4 + D * vbits / 8 + 4) / 4 + D / 32 + 1;   // room for a sketch
  }
  // the staged slots' rows are (swords rounded up to 4) words apart at most
  static __host__ __device__ constexpr int misc_per_warp(int swords) {
    return 16 + 2 * G::ROWS * 8 + 2 * 2 * G::ROWS * 8 + G::ROWS * ((swords + 3) / 4) * 16;
  }
  static __host__ __device__ constexpr int bytes(int kbits, int vbits) {
    return TABLES + 1024 + kAppendWarps * (2 * KIND + misc_per_warp(slot_words(kbits, vbits)));
  }
};

// Quantize-append.  A warp owns tiles of ROWS consecutive (token, KV head) pairs and
// does both halves of each: the K rows, then the V rows (each row: D/64 lanes, 64
// coordinates a lane), into the tile's slots staged in shared memory; then it stores
// the full slots (whole-slot stores, so every DRAM sector of a slot is written by one
// store pass).  Input rows are staged one half-tile ahead.
// SAFE = false: the fast path (rows of ordinary magnitude); when some row leaves its
// range the kernel raises redo[0].  SAFE = true: launched right after it; every CTA
// returns at once unless redo[0] is set, and otherwise the whole call is done again
// with the rescaling rotation (identical results for the other rows); the last CTA
// clears redo.
// QJL: the K rows also store the QJL sketch of their residual (K region: codes, norm,
// D sign bits, residual norm).  FIXB > 0: both code widths are FIXB, fixed at compile
// time (no dispatch on the width in the loop).
template <int D, typename Tin, bool SAFE, bool QJL, int FIXB = 0>
__global__ void __launch_bounds__(kAppendWarps * 32, 2)
append_kernel(AppendParams p, const __grid_constant__ AppendMaps maps) {
  if constexpr (SAFE) {
    if (*(volatile unsigned int*)&p.redo[0] == 0u) return;
  }
  using G = AppendGeom<D>;
  using SM = AppendSmem<D, Tin>;
  extern __shared__ __align__(16) uint8_t smem[];
  EncodeTables* tabs = (EncodeTables*)smem;                       // [2]: K, V
  uint32_t* smask = (uint32_t*)(smem + 2 * sizeof(EncodeTables));  // D sign masks
  int* fast = (int*)(smask + D);                                    // [2] bucket encode valid
  float* kcent_s = (float*)(fast + 4);                              // [256] K centroids (QJL)
  uint32_t* qmask = (uint32_t*)(kcent_s + 256);                     // [D] QJL sketch signs
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kwords = (D * p.bits[0] + 7) / 8 / 4 + 1 + (QJL ? D / 32 + 1 : 0);   // K region
  const int vwords = (D * p.bits[1] + 7) / 8 / 4 + 1;
  const int swords = kwords + vwords;                              // slot words written
  const uint32_t sbase = smem_u32(smem);
  const uint32_t in_off = ((sbase + SM::TABLES + 1023u) & ~1023u) - sbase;
  uint8_t* in_s = smem + in_off + warp * 2 * SM::KIND;             // [2 kinds][KIND]
  uint8_t* misc = smem + in_off + kAppendWarps * 2 * SM::KIND + warp * SM::misc_per_warp(swords);
  uint64_t* bars = (uint64_t*)misc;                                // [2 kinds]
  int64_t* dst_s = (int64_t*)(misc + 16);                          // [2 tiles][ROWS] slots
  const uint8_t** src_s = (const uint8_t**)(dst_s + 2 * G::ROWS);  // [2 tiles][2 kinds][ROWS]
  uint32_t* out_s = (uint32_t*)(src_s + 2 * 2 * G::ROWS);          // [ROWS][srow]
  // words between the staged slots: 16-byte rows when slots are stored one by one
  const int srow = p.slot_body > 0 ? (swords + 3) & ~3 : swords;

  const int64_t npairs = p.num_tokens * p.h_kv;                    // < 2^31 (host check)
  const int64_t ntiles = (npairs + G::ROWS - 1) / G::ROWS;
  const int64_t gwarp = (int64_t)blockIdx.x * kAppendWarps + warp;
  const int64_t nwarps = (int64_t)gridDim.x * kAppendWarps;

  if (lane == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // Resolve tile `tile` (slot offsets; for cp.async staging also the K and V row
  // addresses; lane r < ROWS handles pair r0 + r) into slot `tb`.
  auto resolve = [&](int64_t tile, int tb) {
    const int r0 = (int)(tile * G::ROWS);
    const int nr = (int)imin64((int64_t)G::ROWS, npairs - r0);
    if (lane < nr) {
      const uint32_t row = (uint32_t)(r0 + lane);
      const uint32_t t = row / (uint32_t)p.h_kv;
      const uint32_t h = row - t * (uint32_t)p.h_kv;
      if (!p.tma_in) {
#pragma unroll
        for (int kind = 0; kind < 2; ++kind)
          src_s[(tb * 2 + kind) * G::ROWS + lane] =
              (const uint8_t*)p.src[kind] +
              ((int64_t)t * p.tok_stride[kind] + (int64_t)h * p.head_stride_in[kind]) * SM::RB / D;
      }
      const int64_t slot = p.slot_mapping[(int64_t)t * p.slot_map_stride];
      int64_t off = -1;
      if (slot >= 0) {
        if (slot < p.num_slots) {
          int64_t blk, rr;
          if (p.bs_shift >= 0) {
            blk = slot >> p.bs_shift;
            rr = slot & ((1 << p.bs_shift) - 1);
          } else {
            blk = slot / p.block_size;
            rr = slot - blk * p.block_size;
          }
          off = blk * p.blk_stride + rr * p.row_stride + h * p.head_stride;
        } else {
          report_error(p.err, TQ_DEVERR_SLOT_RANGE);
        }
      }
      dst_s[tb * G::ROWS + lane] = off;
    }
    __syncwarp();
  };
  // Start staging the `kind` rows of the tile resolved in slot tb into buffer `kind`.
  auto stage = [&](int64_t tile, int tb, int kind) {
    uint8_t* buf = in_s + kind * SM::KIND;
    if (p.tma_in) {
      if (lane == 0) {
        const int r0 = (int)(tile * G::ROWS);
        const int t0 = r0 / p.h_kv;
        const int h0 = r0 - t0 * p.h_kv;
        const CUtensorMap* map = kind ? &maps.v : &maps.k;
        mbar_arrive_expect_tx(&bars[kind], SM::KIND);
#pragma unroll
        for (int part = 0; part < G::TPR; ++part)
          tensor_g2s_3d(buf + part * G::ROWS * SM::PB, map, 64 * part, h0, t0, &bars[kind]);
      }
    } else {
      const int nr = (int)imin64((int64_t)G::ROWS, npairs - tile * G::ROWS);
      stage_rows<SM::RB, SM::PB, G::ROWS>(
          buf, nr, [&](int r) { return (const void*)src_s[(tb * 2 + kind) * G::ROWS + r]; },
          p.align_mode, lane);
    }
  };
  // the first tile's K rows are in flight while the tables are built
  if (gwarp < ntiles) {
    resolve(gwarp, 0);
    stage(gwarp, 0, 0);
  }
  cp_async_commit();
  build_tables(&tabs[0], p.boundaries[0], p.bits[0], threadIdx.x, blockDim.x, &fast[0]);
  build_tables(&tabs[1], p.boundaries[1], p.bits[1], threadIdx.x, blockDim.x, &fast[1]);
  for (int j = threadIdx.x; j < D; j += blockDim.x) smask[j] = sign_mask_at(p.sign_seed, j);
  if constexpr (QJL) {
    for (int j = threadIdx.x; j < D; j += blockDim.x) qmask[j] = sign_mask_at(p.qjl_seed, j);
    for (int j = threadIdx.x; j < (1 << p.bits[0]); j += blockDim.x) kcent_s[j] = p.kcent[j];
  }
  __syncthreads();
  build_bucket_table(&tabs[0], p.bits[0], threadIdx.x, blockDim.x);
  build_bucket_table(&tabs[1], p.bits[1], threadIdx.x, blockDim.x);
  __syncthreads();

  const int rl = lane % G::ROWS;           // row within the tile
  const int part = lane / G::ROWS;         // which 64 coordinates of the row
  // this lane's part row in buffer 0, with its swizzle in bits 4-6
  const uint32_t row0 = smem_u32(in_s) + (uint32_t)((part * G::ROWS + rl) * SM::PB) +
                        (uint32_t)((rl & 7) << 4);
  int tb = 0;
  bool redo_needed = false;                 // a row of this lane left the fast path's range
  uint32_t it = 0;                          // tiles done by this warp (mbarrier phase)
  uint32_t staged[2] = {gwarp < ntiles ? 1u : 0u, 0u};   // tensor copies issued per kind
  bool dead = false;
  for (int64_t tile = gwarp; tile < ntiles && !dead; tile += nwarps, ++it) {
    const int nr = (int)imin64((int64_t)G::ROWS, npairs - tile * G::ROWS);
    const int64_t next = tile + nwarps;
#pragma unroll 1
    for (int kind = 0; kind < 2; ++kind) {
      // prefetch one half-tile ahead: this tile's V rows, or the next tile's K rows
      if (kind == 0) {
        stage(tile, tb, 1);
        ++staged[1];
      } else if (next < ntiles) {
        resolve(next, tb ^ 1);
        stage(next, tb ^ 1, 0);
        ++staged[0];
      }
      cp_async_commit();
      if (p.tma_in) {
        const bool ok = mbar_wait(&bars[kind], it & 1u, kWaitMs);
        if (!__all_sync(0xffffffffu, ok)) {     // the warp gives up together
          if (lane == 0) report_error(p.err, TQ_DEVERR_TIMEOUT);
          dead = true;
          break;
        }
      } else {
        cp_async_wait<1>();
      }
      __syncwarp();
      const int bits = p.bits[kind];
      uint64_t xp[32];
      float n;
      bool bad, oor;
      const float r = rotate_row<D, Tin, SAFE>(xp, row0 + (uint32_t)(kind * SM::KIND),
                                               smask + part * 64, part, &n, &bad, &oor);
      if constexpr (!SAFE) redo_needed |= oor && rl < nr;
      if (kind == 0 && (p.bulk_out || p.slot_body > 0)) {   // previous slots read out
        bulk_wait_read_all();
        __syncwarp();
      }
      uint32_t* orow = out_s + rl * srow + (kind ? kwords : 0);
      const EncodeTables* t = &tabs[kind];
      const int cw = D * bits / 32;                        // code words of the region
      const int wpl = cw / G::TPR;                         // code words per lane
      uint32_t* mine = orow + part * wpl;
      const bool sketch = QJL && kind == 0;
      if (!bad) {
        const int use_fast = fast[kind];
        if (sketch) {
          encode_pack_bits<true>(bits, xp, r, t, use_fast, mine, smem_u32(kcent_s));
          uint32_t z0, z1;
          const float gamma = qjl_sketch_row<D>(xp, qmask + part * 64, part, &z0, &z1);
          orow[cw + 1 + 2 * part] = z0;
          orow[cw + 2 + 2 * part] = z1;
          if (part == G::TPR - 1) orow[cw + 1 + D / 32] = __float_as_uint(gamma);
        } else if constexpr (FIXB > 0) {
          encode_pack_any<FIXB, false>(xp, r, t, use_fast, mine, 0u);
        } else {
          encode_pack_bits<false>(bits, xp, r, t, use_fast, mine, 0u);
        }
      } else {
        for (int w = 0; w < wpl; ++w) mine[w] = 0u;
        if (sketch) {
          orow[cw + 1 + 2 * part] = 0u;
          orow[cw + 2 + 2 * part] = 0u;
          if (part == G::TPR - 1) orow[cw + 1 + D / 32] = 0u;
        }
        if (part == 0 && rl < nr) report_error(p.err, TQ_DEVERR_NONFINITE);
      }
      if (part == G::TPR - 1) orow[cw] = bad ? 0x7FC00000u : __float_as_uint(n);
      __syncwarp();
    }
    if (dead) break;
    if (p.bulk_out) {
      // one bulk store per token run of the tile (its heads' slots are contiguous)
      fence_proxy_async_smem();
      __syncwarp();
      const int hr = p.run_heads;
      if (lane * hr < nr) {
        const int64_t off = dst_s[tb * G::ROWS + lane * hr];
        if (off >= 0)
          bulk_s2g(p.pages + off, out_s + lane * hr * swords, (uint32_t)(hr * swords * 4));
        bulk_commit();
      }
    } else if (p.slot_body > 0) {
      // slots one by one (a padded slot stride): each row's 16-byte body by a bulk copy,
      // its tail words by plain stores; the padding is never written
      fence_proxy_async_smem();
      __syncwarp();
      if (lane < nr) {
        const int64_t off = dst_s[tb * G::ROWS + lane];
        if (off >= 0) bulk_s2g(p.pages + off, out_s + lane * srow, (uint32_t)p.slot_body);
        bulk_commit();
      }
      const int bw = p.slot_body >> 2, tw = swords - bw;   // body and tail words
      for (int i = lane; i < nr * tw; i += 32) {
        const int rr = i / tw, w = bw + (i - rr * tw);
        const int64_t off = dst_s[tb * G::ROWS + rr];
        if (off >= 0) ((uint32_t*)(p.pages + off))[w] = out_s[rr * srow + w];
      }
      __syncwarp();
    } else {
      // write back the tile's full slots: lanes run over (pair, word)
      int rr = 0, w = lane;
      while (w >= swords) { w -= swords; ++rr; }
      for (; rr < nr;) {
        const int64_t off = dst_s[tb * G::ROWS + rr];
        if (off >= 0) ((uint32_t*)(p.pages + off))[w] = out_s[rr * swords + w];
        w += 32;
        while (w >= swords) { w -= swords; ++rr; }
      }
      __syncwarp();
    }
    tb ^= 1;
  }
  cp_async_wait<0>();
  if (p.tma_in && dead) {
    // let the tensor copies still in flight land before the CTA's shared memory goes
    // (each kind's copies complete in order; `it` of them were consumed or abandoned)
    for (int kind = 0; kind < 2; ++kind)
      for (uint32_t c = it; c < staged[kind]; ++c)
        if (!mbar_wait(&bars[kind], c & 1u, kWaitMs)) break;
  }
  bulk_wait_all();
  if constexpr (!SAFE) {
    if (__any_sync(0xffffffffu, redo_needed) && lane == 0) atomicExch(&p.redo[0], 1u);
  } else {
    // the last CTA of the redo clears the flag (every CTA has read it by then)
    __syncthreads();
    if (threadIdx.x == 0 && atomicAdd(&p.redo[1], 1u) == gridDim.x - 1) {
      atomicExch(&p.redo[0], 0u);
      atomicExch(&p.redo[1], 0u);
    }
  }
}

// Test export: the rotation of tq_quantize_append, written out as fp32 u and n.
template <int D, typename Tin>
__global__ void __launch_bounds__(kAppendWarps * 32)
rotate_unit_kernel(RotateParams p) {
  using G = AppendGeom<D>;
  using SM = AppendSmem<D, Tin>;
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* smask = (uint32_t*)smem;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t in_off = ((sbase + 4 * D + 1023u) & ~1023u) - sbase;
  uint8_t* in_s = smem + in_off + warp * SM::KIND;
  for (int j = threadIdx.x; j < D; j += blockDim.x) smask[j] = sign_mask_at(p.sign_seed, j);
  __syncthreads();
  const int rl = lane % G::ROWS, part = lane / G::ROWS;
  const uint32_t row = smem_u32(in_s) + (uint32_t)((part * G::ROWS + rl) * SM::PB) +
                       (uint32_t)((rl & 7) << 4);
  const int64_t ntiles = (p.rows + G::ROWS - 1) / G::ROWS;
  for (int64_t tile = (int64_t)blockIdx.x * kAppendWarps + warp; tile < ntiles;
       tile += (int64_t)gridDim.x * kAppendWarps) {
    const int64_t r0 = tile * G::ROWS;
    const int nr = (int)imin64((int64_t)G::ROWS, p.rows - r0);
    const Tin* base = (const Tin*)p.x;
    stage_rows<SM::RB, SM::PB, G::ROWS>(
        in_s, nr, [&](int r) { return (const void*)(base + (r0 + r) * p.x_row_stride); },
        p.align_mode, lane);
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
    uint64_t xp[32];
    float n;
    bool bad, oor;
    const float r = rotate_row<D, Tin, true>(xp, row, smask + part * 64, part, &n, &bad, &oor);
    if (rl < nr) {
      float* u = p.u + (r0 + rl) * p.u_row_stride + part * 64;
      const uint64_t r2 = f2(r, r);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint64_t u2 = mul2(xp[i], r2);
        u[2 * i] = f2lo(u2);
        u[2 * i + 1] = f2hi(u2);
      }
      if (part == 0) p.norm[(r0 + rl) * p.norm_stride] = bad ? __uint_as_float(0x7FC00000u) : n;
    }
    __syncwarp();
  }
}

}  // namespace tq
