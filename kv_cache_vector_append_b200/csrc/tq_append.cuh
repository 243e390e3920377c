// tq_append.cuh -- quantize-append: rotate, norm, Lloyd-Max encode, bit-pack,
// store into page slots.
//
// Follows TorbuQuant (ginkgoq.github.io/TurboQuant), "TQ4 page tensor" diagram and
// the "Quantize" / "Store" stages; tq-kv (shadowgraph.io), "How It Works" step 3
// (randomized Hadamard transform); turboquant_serve 0.1.2, "Architecture" (update():
// rotate, normalize, Lloyd-Max encode, bit-pack, store uint8).
//
// Work layout.  A row is one (token, KV head) vector of K or of V.  A warp owns a
// tile of 32 rows of one kind (K or V); for D <= 128 each lane holds a whole row in
// registers (no shuffles in the transform), for D = 256 two lanes share a row
// (one cross-lane butterfly stage).  Input tiles are staged in shared memory with
// cp.async (double-buffered per warp) so that global reads are fully coalesced;
// packed regions are staged in shared memory and written back one contiguous
// region per store instruction.
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

constexpr int kAppendWarps = 4;

template <int D>
struct AppendGeom {
  static constexpr int TPR = D > 128 ? D / 128 : 1;   // lanes per row
  static constexpr int E = D / TPR;                   // elements per lane
  static constexpr int ROWS = 32 / TPR;               // rows per warp tile
  static constexpr int MAXW = D * 8 / 32 + 1;         // packed words + norm, 8-bit
  static constexpr int OUTPITCH = MAXW | 1;           // odd pitch: conflict-free
};

// Builds the Eytzinger (breadth-first) image of the sorted boundary array so
// that a binary search walks i -> 2i + (u > t[i]).  t[0] is unused.
__device__ __forceinline__ void build_eytzinger(float* t, const float* b, int bits, int tid,
                                                int nthreads) {
  const int n = (1 << bits) - 1;
  for (int i = 1 + tid; i <= n; i += nthreads) {
    int d = 31 - __clz(i);
    int k = i - (1 << d);
    int src = ((2 * k + 1) << (bits - 1 - d)) - 1;
    t[i] = b[src];
  }
}

// Stage `nrows` rows of `rowbytes` bytes into shared memory (pitch `pitch`).
// Row r starts at row_ptr(r).  Issued by one warp.
template <int D, typename Tin, typename RowPtr>
__device__ __forceinline__ void stage_rows(uint8_t* dst, int pitch, int nrows, RowPtr row_ptr,
                                           int align_mode, int lane) {
  constexpr int RB = D * InType<Tin>::kBytes;
  if (align_mode == 16) {
    constexpr int NC = RB / 16;
    for (int f = lane; f < nrows * NC; f += 32) {
      int r = f / NC, c = f % NC;
      cp_async16(dst + r * pitch + c * 16, (const uint8_t*)row_ptr(r) + c * 16);
    }
  } else if (align_mode == 4) {
    constexpr int NC = RB / 4;
    for (int f = lane; f < nrows * NC; f += 32) {
      int r = f / NC, c = f % NC;
      cp_async4(dst + r * pitch + c * 4, (const uint8_t*)row_ptr(r) + c * 4);
    }
  } else {
    constexpr int NC = RB / 2;
    for (int f = lane; f < nrows * NC; f += 32) {
      int r = f / NC, c = f % NC;
      *(uint16_t*)(dst + r * pitch + c * 2) = *((const uint16_t*)row_ptr(r) + c);
    }
  }
}

// Load this lane's E elements of its row from shared memory as fp32.
template <int E, typename Tin>
__device__ __forceinline__ void load_row(float (&x)[E], const uint8_t* p) {
  if constexpr (sizeof(Tin) == 4) {
#pragma unroll
    for (int c = 0; c < E / 4; ++c) {
      float4 q = *(const float4*)(p + 16 * c);
      x[4 * c + 0] = q.x; x[4 * c + 1] = q.y; x[4 * c + 2] = q.z; x[4 * c + 3] = q.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < E / 8; ++c) {
      uint4 q = *(const uint4*)(p + 16 * c);
      uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if constexpr (std::is_same<Tin, __nv_bfloat16>::value) {
          x[8 * c + 2 * k + 0] = __uint_as_float(w[k] << 16);
          x[8 * c + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
        } else {
          __half2 h = *reinterpret_cast<__half2*>(&w[k]);
          float2 f = __half22float2(h);
          x[8 * c + 2 * k + 0] = f.x;
          x[8 * c + 2 * k + 1] = f.y;
        }
      }
    }
  }
}

// The rotation shared by quantize-append and its test export.  On entry x holds
// this lane's E input elements (coordinates half*E .. half*E+E-1 of the row); on
// exit x holds the unnormalised transform H (s * x) of those coordinates, and the
// function returns the scale r with u = x * r; *norm_out = ||x||_2 (fp32).
// Order of operations (fixed, so the export reproduces the kernel exactly):
//   ss = sum of x_j^2 by fused multiply-add in coordinate order (lane pairs then
//   add their halves), n = sqrt(ss) (IEEE), sign flips, FWHT butterflies in
//   stages h = 1, 2, 4, ..., D/2, r = 1 / (n * sqrt(D)) (IEEE reciprocal), or 0
//   when n == 0.
template <int D>
__device__ __forceinline__ float rotate_row(float (&x)[AppendGeom<D>::E], const uint32_t* smask,
                                            int half, float* norm_out) {
  constexpr int E = AppendGeom<D>::E;
  constexpr int TPR = AppendGeom<D>::TPR;
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < E; ++j) ss = __fmaf_rn(x[j], x[j], ss);
  if constexpr (TPR == 2) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, 1));
  const float n = sqrtf(ss);
#pragma unroll
  for (int c = 0; c < E / 4; ++c) {
    uint4 m = *(const uint4*)(smask + half * E + 4 * c);
    x[4 * c + 0] = __uint_as_float(__float_as_uint(x[4 * c + 0]) ^ m.x);
    x[4 * c + 1] = __uint_as_float(__float_as_uint(x[4 * c + 1]) ^ m.y);
    x[4 * c + 2] = __uint_as_float(__float_as_uint(x[4 * c + 2]) ^ m.z);
    x[4 * c + 3] = __uint_as_float(__float_as_uint(x[4 * c + 3]) ^ m.w);
  }
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int i = 0; i < E; ++i) {
      if ((i & h) == 0) {
        float a = x[i], b = x[i + h];
        x[i] = __fadd_rn(a, b);
        x[i + h] = __fsub_rn(a, b);
      }
    }
  }
  if constexpr (TPR == 2) {
#pragma unroll
    for (int i = 0; i < E; ++i) {
      float o = __shfl_xor_sync(0xffffffffu, x[i], 1);
      x[i] = half == 0 ? __fadd_rn(x[i], o) : __fsub_rn(o, x[i]);
    }
  }
  *norm_out = n;
  const float sqrt_d = D == 64 ? 8.0f : (D == 128 ? 11.313708498984761f : 16.0f);
  return n > 0.f ? __frcp_rn(__fmul_rn(n, sqrt_d)) : 0.f;
}

// Encode u = x[j] * r with the Eytzinger table and pack the codes LSB-first into
// `words` (E*BITS/32 words: this lane's share of the bit stream).
template <int E, int BITS>
__device__ __forceinline__ void encode_pack(const float (&x)[E], float r, const float* tab,
                                            uint32_t* words) {
  constexpr int W = E * BITS / 32;
  uint32_t acc[W];
#pragma unroll
  for (int w = 0; w < W; ++w) acc[w] = 0u;
#pragma unroll
  for (int j = 0; j < E; ++j) {
    const float u = __fmul_rn(x[j], r);
    int i = 1;
#pragma unroll
    for (int s = 0; s < BITS; ++s) i = 2 * i + (u > tab[i] ? 1 : 0);
    const uint32_t code = (uint32_t)(i - (1 << BITS));
    constexpr int dummy = 0;
    (void)dummy;
    const int bit = j * BITS;
    const int w0 = bit >> 5, o0 = bit & 31;
    acc[w0] |= code << o0;
    if (o0 + BITS > 32) acc[w0 + 1] |= code >> (32 - o0);
  }
#pragma unroll
  for (int w = 0; w < W; ++w) words[w] = acc[w];
}

template <int D, typename Tin>
__global__ void __launch_bounds__(kAppendWarps * 32)
append_kernel(AppendParams p) {
  using G = AppendGeom<D>;
  constexpr int RB = D * InType<Tin>::kBytes;
  constexpr int INPITCH = RB + 16;
  extern __shared__ __align__(16) uint8_t smem[];
  float* tab = (float*)smem;                           // 2 x 256 floats (Eytzinger, K and V)
  uint32_t* smask = (uint32_t*)(smem + 2048);          // D sign masks
  uint8_t* wbase = smem + 2048 + 4 * D;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int PER_WARP = 2 * G::ROWS * INPITCH + G::ROWS * G::OUTPITCH * 4 + G::ROWS * 8;
  uint8_t* in_s = wbase + warp * PER_WARP;
  uint32_t* out_s = (uint32_t*)(in_s + 2 * G::ROWS * INPITCH);
  int64_t* dst_s = (int64_t*)(out_s + G::ROWS * G::OUTPITCH);

  build_eytzinger(tab, p.boundaries[0], p.bits[0], threadIdx.x, blockDim.x);
  build_eytzinger(tab + 256, p.boundaries[1], p.bits[1], threadIdx.x, blockDim.x);
  for (int j = threadIdx.x; j < D; j += blockDim.x) smask[j] = sign_mask_at(p.sign_seed, j);
  __syncthreads();

  const int64_t rows_per_kind = p.num_tokens * p.h_kv;
  const int64_t tiles_per_kind = (rows_per_kind + G::ROWS - 1) / G::ROWS;
  const int64_t ntiles = 2 * tiles_per_kind;
  const int64_t gwarp = (int64_t)blockIdx.x * kAppendWarps + warp;
  const int64_t nwarps = (int64_t)gridDim.x * kAppendWarps;

  auto issue = [&](int64_t tile, int buf) {
    const int kind = tile >= tiles_per_kind;
    const int64_t r0 = (tile - kind * tiles_per_kind) * G::ROWS;
    const int nr = (int)imin64((int64_t)G::ROWS, rows_per_kind - r0);
    const Tin* base = (const Tin*)p.src[kind];
    const int64_t ts = p.tok_stride[kind], hs = p.head_stride_in[kind];
    const int hk = p.h_kv;
    stage_rows<D, Tin>(in_s + buf * G::ROWS * INPITCH, INPITCH, nr,
                       [&](int r) {
                         int64_t row = r0 + r;
                         int64_t t = row / hk;
                         int h = (int)(row - t * hk);
                         return (const void*)(base + t * ts + h * hs);
                       },
                       p.align_mode, lane);
  };

  int buf = 0;
  if (gwarp < ntiles) issue(gwarp, 0);
  cp_async_commit();
  for (int64_t tile = gwarp; tile < ntiles; tile += nwarps) {
    const int64_t next = tile + nwarps;
    if (next < ntiles) issue(next, buf ^ 1);
    cp_async_commit();
    const int kind = tile >= tiles_per_kind;
    const int64_t r0 = (tile - kind * tiles_per_kind) * G::ROWS;
    const int nr = (int)imin64((int64_t)G::ROWS, rows_per_kind - r0);
    const int bits = p.bits[kind];
    const int nw = D * bits / 32 + 1;   // packed words + norm word
    // destination byte offset of each row's region (-1: skip)
    if (lane < nr) {
      const int64_t row = r0 + lane;
      const int64_t t = row / p.h_kv;
      const int h = (int)(row - t * p.h_kv);
      const int64_t slot = p.slot_mapping[t * p.slot_map_stride];
      int64_t off = -1;
      if (slot >= 0) {
        if (slot < p.num_slots) {
          const int64_t blk = slot / p.block_size, rr = slot - blk * p.block_size;
          off = blk * p.blk_stride + rr * p.row_stride + h * p.head_stride + p.region_off[kind];
        } else {
          report_error(p.err, TQ_DEVERR_SLOT_RANGE);
        }
      }
      dst_s[lane] = off;
    }
    cp_async_wait<1>();
    __syncwarp();
    {
      const int rl = lane / G::TPR;          // row within the tile
      const int half = lane % G::TPR;
      float x[G::E];
      load_row<G::E, Tin>(x, in_s + buf * G::ROWS * INPITCH + rl * INPITCH + half * G::E *
                                  InType<Tin>::kBytes);
      float n;
      const float r = rotate_row<D>(x, smask, half, &n);
      const bool bad = !(fabsf(n) <= 3.402823466e38f);   // inf or NaN
      uint32_t* orow = out_s + rl * G::OUTPITCH;
      const float* t = tab + 256 * kind;
      const int wpl = (nw - 1) / G::TPR;                  // words per lane
      uint32_t* mine = orow + half * wpl;
      switch (bits) {
        case 1: encode_pack<G::E, 1>(x, r, t, mine); break;
        case 2: encode_pack<G::E, 2>(x, r, t, mine); break;
        case 3: encode_pack<G::E, 3>(x, r, t, mine); break;
        case 4: encode_pack<G::E, 4>(x, r, t, mine); break;
        case 5: encode_pack<G::E, 5>(x, r, t, mine); break;
        case 6: encode_pack<G::E, 6>(x, r, t, mine); break;
        case 7: encode_pack<G::E, 7>(x, r, t, mine); break;
        default: encode_pack<G::E, 8>(x, r, t, mine); break;
      }
      if (bad) {
        for (int w = 0; w < wpl; ++w) mine[w] = 0u;
        if (half == 0 && rl < nr) report_error(p.err, TQ_DEVERR_NONFINITE);
      }
      if (half == G::TPR - 1) orow[nw - 1] = bad ? 0x7FC00000u : __float_as_uint(n);
    }
    __syncwarp();
    // write back: one row region per pass (contiguous words)
    for (int rr = 0; rr < nr; ++rr) {
      const int64_t off = dst_s[rr];
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

template <int D>
constexpr size_t append_smem_bytes(int in_bytes) {
  using G = AppendGeom<D>;
  return 2048 + 4 * D +
         (size_t)kAppendWarps * (2 * G::ROWS * (D * in_bytes + 16) + G::ROWS * G::OUTPITCH * 4 +
                                 G::ROWS * 8);
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
  const int64_t ntiles = (p.rows + G::ROWS - 1) / G::ROWS;
  for (int64_t tile = (int64_t)blockIdx.x * kAppendWarps + warp; tile < ntiles;
       tile += (int64_t)gridDim.x * kAppendWarps) {
    const int64_t r0 = tile * G::ROWS;
    const int nr = (int)imin64((int64_t)G::ROWS, p.rows - r0);
    const Tin* base = (const Tin*)p.x;
    stage_rows<D, Tin>(in_s, INPITCH, nr,
                       [&](int r) { return (const void*)(base + (r0 + r) * p.x_row_stride); },
                       p.align_mode, lane);
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
    const int rl = lane / G::TPR, half = lane % G::TPR;
    float x[G::E];
    load_row<G::E, Tin>(x, in_s + rl * INPITCH + half * G::E * InType<Tin>::kBytes);
    float n;
    const float r = rotate_row<D>(x, smask, half, &n);
    if (rl < nr) {
      float* u = p.u + (r0 + rl) * p.u_row_stride + half * G::E;
#pragma unroll
      for (int j = 0; j < G::E; ++j) u[j] = __fmul_rn(x[j], r);
      if (half == 0) p.norm[(r0 + rl) * p.norm_stride] = n;
    }
    __syncwarp();
  }
}

}  // namespace tq
