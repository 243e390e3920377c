// tq_append.cuh -- quantize-append: rotate, norm, Lloyd-Max encode, bit-pack,
// store into page slots.
//
// Follows TorbuQuant (ginkgoq.github.io/TurboQuant), "TQ4 page tensor" diagram and
// the "Quantize" / "Store" stages; tq-kv (shadowgraph.io), "How It Works" step 3
// (randomized Hadamard transform); turboquant_serve 0.1.2, "Architecture" (update():
// rotate, normalize, Lloyd-Max encode, bit-pack, store uint8).
//
// Work layout.  A row is one (token, KV head) vector of K or of V.  Every lane holds
// 64 consecutive coordinates of a row in registers (D/64 lanes per row), so the FWHT
// is six register stages plus log2(D/64) shuffle stages.  A warp owns a tile of
// 32*64/D rows of one kind (K or V); lane l serves row l % ROWS, part l / ROWS, so
// that each 8-lane phase of a 16-byte shared load touches 8 different rows (padded
// pitch, no bank conflicts).  Input tiles are staged in shared memory by cp.async
// (double-buffered per warp); packed regions are staged in shared memory and
// written back one contiguous region per store instruction.
//
// Encode.  idx = #{i : b_i < u} over the fp32 boundaries.  For bits <= 4 (and when no
// two boundaries share a bucket) the top 12 bits of u's float encoding (sign,
// exponent, 3 mantissa bits) index a byte table k0 = #{b_i < lowest float of the
// bucket}; one compare against b[k0] then gives idx exactly.  Otherwise a
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
  static constexpr int MAXW = D * 8 / 32 + 1;         // packed words + norm, 8-bit
  static constexpr int OUTPITCH = MAXW | 1;           // odd pitch: conflict-free
};

// Shared tables of one kind (K or V).
struct alignas(16) EncodeTables {
  uint8_t k0[kBuckets];     // #{b_i < lowest float of the bucket}
  float bnd[257];           // boundaries b_0..b_{L-2}, then +inf
  float eytz[256];          // Eytzinger image (t[0] unused)
  int fast;                 // bucket encode valid for this table
};

// Phase 1 (then a CTA barrier, then phase 2): boundaries, Eytzinger image, and the
// check that no two boundaries share a bucket.
__device__ __forceinline__ void build_tables(EncodeTables* t, const float* b, int bits, int tid,
                                             int nthreads) {
  const int n = (1 << bits) - 1;
  for (int i = tid; i <= n; i += nthreads) t->bnd[i] = i < n ? b[i] : INFINITY;
  for (int i = 1 + tid; i <= n; i += nthreads) {
    const int d = 31 - __clz(i);
    const int k = i - (1 << d);
    t->eytz[i] = b[((2 * k + 1) << (bits - 1 - d)) - 1];
  }
  if (tid == 0) {
    int ok = bits <= 4;
    for (int i = 0; i + 1 < n; ++i)
      if ((__float_as_uint(b[i]) >> kBucketShift) == (__float_as_uint(b[i + 1]) >> kBucketShift))
        ok = 0;
    t->fast = ok;
  }
}

// Phase 2: k0 of each bucket = #{b_i < lowest float of the bucket}, by binary search
// over the boundaries already in shared memory.  The lowest float of bucket g is
// g << 20 for a positive bucket and -((g & 0x7ff) << 20 | 0xfffff) for a negative one.
// Only used for bits <= 4.
__device__ __forceinline__ void build_bucket_table(EncodeTables* t, int bits, int tid,
                                                   int nthreads) {
  if (bits > 4) return;
  const int n = (1 << bits) - 1;
  for (int g = tid; g < kBuckets; g += nthreads) {
    const uint32_t lowbits = (g & 0x800) ? ((uint32_t)g << kBucketShift) | 0xFFFFFu
                                         : (uint32_t)g << kBucketShift;
    const float lo = __uint_as_float(lowbits);
    int a = 0, c = n;                   // count of boundaries < lo lies in [a, c]
    while (a < c) {
      const int m = (a + c) >> 1;
      if (t->bnd[m] < lo) a = m + 1; else c = m;
    }
    t->k0[g] = (uint8_t)a;
  }
}

// Stage `nrows` rows of RB bytes into shared memory (pitch `pitch`); row r starts at
// row_ptr(r).  Issued by one warp.
template <int RB, typename RowPtr>
__device__ __forceinline__ void stage_rows(uint8_t* dst, int pitch, int nrows, RowPtr row_ptr,
                                           int align_mode, int lane) {
  if (align_mode == 16) {
    constexpr int NC = RB / 16;
    for (int f = lane; f < nrows * NC; f += 32) {
      const int r = f / NC, c = f % NC;
      cp_async16(dst + r * pitch + c * 16, (const uint8_t*)row_ptr(r) + c * 16);
    }
  } else if (align_mode == 4) {
    constexpr int NC = RB / 4;
    for (int f = lane; f < nrows * NC; f += 32) {
      const int r = f / NC, c = f % NC;
      cp_async4(dst + r * pitch + c * 4, (const uint8_t*)row_ptr(r) + c * 4);
    }
  } else {
    constexpr int NC = RB / 2;
    for (int f = lane; f < nrows * NC; f += 32) {
      const int r = f / NC, c = f % NC;
      *(uint16_t*)(dst + r * pitch + c * 2) = *((const uint16_t*)row_ptr(r) + c);
    }
  }
}

// Load this lane's 64 input elements from shared memory as fp32 with the rotation
// signs applied (the sign flip is an xor of the sign bit; for bf16 it rides along
// with the widening: bits << 16 plus the mask, or the high half masked and xor-ed).
template <typename Tin>
__device__ __forceinline__ void load_signed(float (&x)[64], const uint8_t* p,
                                            const uint32_t* m) {
  if constexpr (sizeof(Tin) == 4) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const uint4 q = *(const uint4*)(p + 16 * c);
      const uint4 s = *(const uint4*)(m + 4 * c);
      x[4 * c + 0] = __uint_as_float(q.x ^ s.x);
      x[4 * c + 1] = __uint_as_float(q.y ^ s.y);
      x[4 * c + 2] = __uint_as_float(q.z ^ s.z);
      x[4 * c + 3] = __uint_as_float(q.w ^ s.w);
    }
  } else {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 q = *(const uint4*)(p + 16 * c);
      const uint4 s0 = *(const uint4*)(m + 8 * c);
      const uint4 s1 = *(const uint4*)(m + 8 * c + 4);
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
      const uint32_t s[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if constexpr (std::is_same<Tin, __nv_bfloat16>::value) {
          x[8 * c + 2 * k + 0] = __uint_as_float((w[k] << 16) ^ s[2 * k]);
          x[8 * c + 2 * k + 1] = __uint_as_float((w[k] & 0xFFFF0000u) ^ s[2 * k + 1]);
        } else {
          __half2 h = *reinterpret_cast<const __half2*>(&w[k]);
          const float2 f = __half22float2(h);
          x[8 * c + 2 * k + 0] = __uint_as_float(__float_as_uint(f.x) ^ s[2 * k]);
          x[8 * c + 2 * k + 1] = __uint_as_float(__float_as_uint(f.y) ^ s[2 * k + 1]);
        }
      }
    }
  }
}

// The rotation shared by quantize-append and its test export.  On entry x holds
// this lane's 64 sign-flipped input elements (coordinates 64*part .. 64*part+63 of
// the row); on exit x holds the unnormalised transform H (s * x) of those
// coordinates, and the function returns r with u = x * r; *norm_out = ||x||_2.
// Order of operations (fixed, so the export reproduces the kernel exactly):
//   ss = sum of x_j^2 by fused multiply-add in coordinate order within a lane, then
//   the lanes of a row add their sums pairwise (xor butterfly over the part bits);
//   n = sqrt(ss) (IEEE); FWHT butterflies in stages h = 1, 2, 4, ..., D/2;
//   r = 1 / (n * sqrt(D)) (IEEE reciprocal), or 0 when n == 0.
template <int D>
__device__ __forceinline__ float rotate_row(float (&x)[64], int part, float* norm_out) {
  using G = AppendGeom<D>;
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < 64; ++j) ss = __fmaf_rn(x[j], x[j], ss);
#pragma unroll
  for (int m = 1; m < G::TPR; m <<= 1)
    ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, G::ROWS * m));
  const float n = sqrtf(ss);
#pragma unroll
  for (int h = 1; h < 64; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      if ((i & h) == 0) {
        const float a = x[i], b = x[i + h];
        x[i] = __fadd_rn(a, b);
        x[i + h] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int m = 1; m < G::TPR; m <<= 1) {
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, x[i], G::ROWS * m);
      x[i] = (part & m) ? __fsub_rn(o, x[i]) : __fadd_rn(x[i], o);
    }
  }
  *norm_out = n;
  const float sqrt_d = D == 64 ? 8.0f : (D == 128 ? 11.313708498984761f : 16.0f);
  return n > 0.f ? __frcp_rn(__fmul_rn(n, sqrt_d)) : 0.f;
}

// Encode u = x[j] * r and pack the 64 codes LSB-first into 2*BITS words.
template <int BITS, bool FAST>
__device__ __forceinline__ void encode_pack(const float (&x)[64], float r, const EncodeTables* t,
                                            uint32_t* words) {
  constexpr int W = 64 * BITS / 32;
  uint32_t acc[W];
#pragma unroll
  for (int w = 0; w < W; ++w) acc[w] = 0u;
#pragma unroll
  for (int j = 0; j < 64; ++j) {
    const float u = __fmul_rn(x[j], r);
    uint32_t code;
    if constexpr (FAST) {
      const uint32_t k0 = t->k0[__float_as_uint(u) >> kBucketShift];
      code = k0 + (u > t->bnd[k0] ? 1u : 0u);
    } else {
      int i = 1;
#pragma unroll
      for (int s = 0; s < BITS; ++s) i = 2 * i + (u > t->eytz[i] ? 1 : 0);
      code = (uint32_t)(i - (1 << BITS));
    }
    const int bit = j * BITS;
    const int w0 = bit >> 5, o0 = bit & 31;
    acc[w0] |= code << o0;
    if (o0 + BITS > 32) acc[w0 + 1] |= code >> (32 - o0);
  }
#pragma unroll
  for (int w = 0; w < W; ++w) words[w] = acc[w];
}

template <int BITS>
__device__ __forceinline__ void encode_pack_any(const float (&x)[64], float r,
                                                const EncodeTables* t, uint32_t* words) {
  if constexpr (BITS <= 4) {
    if (t->fast) {
      encode_pack<BITS, true>(x, r, t, words);
      return;
    }
  }
  encode_pack<BITS, false>(x, r, t, words);
}

template <int D, typename Tin>
struct AppendSmem {
  using G = AppendGeom<D>;
  static constexpr int RB = D * InType<Tin>::kBytes;
  static constexpr int INPITCH = RB + 16;
  static constexpr int PER_WARP =
      2 * G::ROWS * INPITCH + G::ROWS * G::OUTPITCH * 4 + 2 * G::ROWS * 8 + 2 * G::ROWS * 8;
  static constexpr int TABLES = ((2 * (int)sizeof(EncodeTables) + 4 * D) + 127) / 128 * 128;
  static constexpr int BYTES = TABLES + kAppendWarps * PER_WARP;
};

template <int D, typename Tin>
__global__ void __launch_bounds__(kAppendWarps * 32, 2)
append_kernel(AppendParams p) {
  using G = AppendGeom<D>;
  using SM = AppendSmem<D, Tin>;
  extern __shared__ __align__(16) uint8_t smem[];
  EncodeTables* tabs = (EncodeTables*)smem;                       // [2]: K, V
  uint32_t* smask = (uint32_t*)(smem + 2 * sizeof(EncodeTables));  // D sign masks
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* in_s = smem + SM::TABLES + warp * SM::PER_WARP;
  uint32_t* out_s = (uint32_t*)(in_s + 2 * G::ROWS * SM::INPITCH);
  int64_t* dst_s = (int64_t*)(out_s + G::ROWS * G::OUTPITCH);     // [2][ROWS] region offsets
  const uint8_t** src_s = (const uint8_t**)(dst_s + 2 * G::ROWS);  // [2][ROWS] row addresses

  const int64_t rows_per_kind = p.num_tokens * p.h_kv;            // < 2^31 (host check)
  const int64_t tiles_per_kind = (rows_per_kind + G::ROWS - 1) / G::ROWS;
  const int64_t ntiles = 2 * tiles_per_kind;
  const int64_t gwarp = (int64_t)blockIdx.x * kAppendWarps + warp;
  const int64_t nwarps = (int64_t)gridDim.x * kAppendWarps;

  // Stage tile `tile` into buffer `buf`: lane r < ROWS resolves row r0 + r once (its
  // input address and its slot's region offset), then the warp copies the rows.
  auto issue = [&](int64_t tile, int buf) {
    const int kind = tile >= tiles_per_kind;
    const int r0 = (int)((tile - kind * tiles_per_kind) * G::ROWS);
    const int nr = (int)imin64((int64_t)G::ROWS, rows_per_kind - r0);
    if (lane < nr) {
      const uint32_t row = (uint32_t)(r0 + lane);
      const uint32_t t = row / (uint32_t)p.h_kv;
      const uint32_t h = row - t * (uint32_t)p.h_kv;
      src_s[buf * G::ROWS + lane] =
          (const uint8_t*)p.src[kind] +
          ((int64_t)t * p.tok_stride[kind] + (int64_t)h * p.head_stride_in[kind]) * SM::RB / D;
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
          off = blk * p.blk_stride + rr * p.row_stride + h * p.head_stride + p.region_off[kind];
        } else {
          report_error(p.err, TQ_DEVERR_SLOT_RANGE);
        }
      }
      dst_s[buf * G::ROWS + lane] = off;
    }
    __syncwarp();
    stage_rows<SM::RB>(in_s + buf * G::ROWS * SM::INPITCH, SM::INPITCH, nr,
                       [&](int r) { return (const void*)src_s[buf * G::ROWS + r]; },
                       p.align_mode, lane);
  };
  // the first tile's rows are in flight while the tables are built
  if (gwarp < ntiles) issue(gwarp, 0);
  cp_async_commit();
  build_tables(&tabs[0], p.boundaries[0], p.bits[0], threadIdx.x, blockDim.x);
  build_tables(&tabs[1], p.boundaries[1], p.bits[1], threadIdx.x, blockDim.x);
  for (int j = threadIdx.x; j < D; j += blockDim.x) smask[j] = sign_mask_at(p.sign_seed, j);
  __syncthreads();
  build_bucket_table(&tabs[0], p.bits[0], threadIdx.x, blockDim.x);
  build_bucket_table(&tabs[1], p.bits[1], threadIdx.x, blockDim.x);
  __syncthreads();

  const int rl = lane % G::ROWS;           // row within the tile
  const int part = lane / G::ROWS;         // which 64 coordinates of the row
  int buf = 0;
  for (int64_t tile = gwarp; tile < ntiles; tile += nwarps) {
    const int64_t next = tile + nwarps;
    if (next < ntiles) issue(next, buf ^ 1);
    cp_async_commit();
    const int kind = tile >= tiles_per_kind;
    const int64_t r0 = (tile - kind * tiles_per_kind) * G::ROWS;
    const int nr = (int)imin64((int64_t)G::ROWS, rows_per_kind - r0);
    const int bits = p.bits[kind];
    const int nw = D * bits / 32 + 1;   // packed words + norm word
    cp_async_wait<1>();
    __syncwarp();
    {
      float x[64];
      load_signed<Tin>(x, in_s + buf * G::ROWS * SM::INPITCH + rl * SM::INPITCH +
                              part * 64 * InType<Tin>::kBytes,
                       smask + part * 64);
      float n;
      const float r = rotate_row<D>(x, part, &n);
      const bool bad = !(fabsf(n) <= 3.402823466e38f);   // inf or NaN
      uint32_t* orow = out_s + rl * G::OUTPITCH;
      const EncodeTables* t = &tabs[kind];
      const int wpl = (nw - 1) / G::TPR;                  // words per lane
      uint32_t* mine = orow + part * wpl;
      switch (bits) {
        case 1: encode_pack_any<1>(x, r, t, mine); break;
        case 2: encode_pack_any<2>(x, r, t, mine); break;
        case 3: encode_pack_any<3>(x, r, t, mine); break;
        case 4: encode_pack_any<4>(x, r, t, mine); break;
        case 5: encode_pack_any<5>(x, r, t, mine); break;
        case 6: encode_pack_any<6>(x, r, t, mine); break;
        case 7: encode_pack_any<7>(x, r, t, mine); break;
        default: encode_pack_any<8>(x, r, t, mine); break;
      }
      if (bad) {
        for (int w = 0; w < wpl; ++w) mine[w] = 0u;
        if (part == 0 && rl < nr) report_error(p.err, TQ_DEVERR_NONFINITE);
      }
      if (part == G::TPR - 1) orow[nw - 1] = bad ? 0x7FC00000u : __float_as_uint(n);
    }
    __syncwarp();
    // write back: one row region per pass (contiguous words)
    for (int rr = 0; rr < nr; ++rr) {
      const int64_t off = dst_s[buf * G::ROWS + rr];
      if (off < 0) continue;
      uint32_t* dst = (uint32_t*)(p.pages + off);
      const uint32_t* src = out_s + rr * G::OUTPITCH;
      for (int w = lane; w < nw; w += 32) dst[w] = src[w];
    }
    __syncwarp();
    buf ^= 1;
  }
  cp_async_wait<0>();
}

// Test export: the rotation of tq_quantize_append, written out as fp32 u and n.
template <int D, typename Tin>
__global__ void __launch_bounds__(kAppendWarps * 32)
rotate_unit_kernel(RotateParams p) {
  using G = AppendGeom<D>;
  constexpr int RB = D * InType<Tin>::kBytes;
  constexpr int INPITCH = RB + 16;
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* smask = (uint32_t*)smem;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* in_s = smem + 4 * D + warp * G::ROWS * INPITCH;
  for (int j = threadIdx.x; j < D; j += blockDim.x) smask[j] = sign_mask_at(p.sign_seed, j);
  __syncthreads();
  const int rl = lane % G::ROWS, part = lane / G::ROWS;
  const int64_t ntiles = (p.rows + G::ROWS - 1) / G::ROWS;
  for (int64_t tile = (int64_t)blockIdx.x * kAppendWarps + warp; tile < ntiles;
       tile += (int64_t)gridDim.x * kAppendWarps) {
    const int64_t r0 = tile * G::ROWS;
    const int nr = (int)imin64((int64_t)G::ROWS, p.rows - r0);
    const Tin* base = (const Tin*)p.x;
    stage_rows<RB>(in_s, INPITCH, nr,
                   [&](int r) { return (const void*)(base + (r0 + r) * p.x_row_stride); },
                   p.align_mode, lane);
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
    float x[64];
    load_signed<Tin>(x, in_s + rl * INPITCH + part * 64 * InType<Tin>::kBytes, smask + part * 64);
    float n;
    const float r = rotate_row<D>(x, part, &n);
    if (rl < nr) {
      float* u = p.u + (r0 + rl) * p.u_row_stride + part * 64;
#pragma unroll
      for (int j = 0; j < 64; ++j) u[j] = __fmul_rn(x[j], r);
      if (part == 0) p.norm[(r0 + rl) * p.norm_stride] = n;
    }
    __syncwarp();
  }
}

}  // namespace tq
