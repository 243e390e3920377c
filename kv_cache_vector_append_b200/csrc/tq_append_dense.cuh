// tq_append_dense.cuh -- quantize-append with the dense random rotation, on the tcgen05
// tensor cores.
//
// Follows turboquant_serve 0.1.2, "Architecture" (rotate: k, v = k @ R; "Rotation": a
// fixed random orthogonal matrix per head_dim), TorbuQuant, "Current Status" (QR and
// RHT rotations) and turboquant_pro 1.4.2, "Fused CUDA decode" (rotate and quantize
// fused into one tiled GEMM).  The rotation R = hi + lo (two bf16 matrices, exact in
// fp32: see the rotation table's file format) replaces the randomized Hadamard
// transform; the norm, encode and slot layout are those of tq_append.cuh.
//
// Work layout.  A tile is 128 consecutive (token, KV head) pairs.  Its K rows and V rows
// (bf16) come in by 3-D tensor copies, 64 elements x heads x tokens per box, with the
// 128-byte swizzle, which is the K-major SWIZZLE_128B operand layout of tcgen05.mma:
// row r of a 64-column block at byte r * 128 of the block, 16-byte chunk c at chunk
// c ^ (r & 7).  R hi and R lo sit in shared memory in the same layout (rows j, columns
// k), so one MMA step computes Y[128 x D] += X[128 x 16] R[D x 16]^T, i.e. y = R x for
// every row, accumulated in fp32 in tensor memory: K rows in columns [0, D), V rows in
// [D, 2D).  One thread issues the copies and the MMAs (D/16 steps x hi, lo per kind);
// the epilogue runs on all eight warps: warps 0-3 take the K rows, warps 4-7 the V rows,
// each thread one row (its lane quarter of tensor memory): the row's norm from the
// staged input, then u = y / n in chunks of 32 columns read with tcgen05.ld, encoded
// and packed into the tile's slots in shared memory, which leave with coalesced stores.
// Input tiles are double-buffered: the copies of tile i+1 run during tile i.
#pragma once

#include "tq_append.cuh"

namespace tq {

struct DenseAppendParams {
  uint8_t* pages;
  int64_t num_slots;
  int32_t block_size;
  int32_t bs_shift;
  int32_t h_kv;
  int64_t blk_stride, row_stride, head_stride;   // bytes
  const int64_t* slot_mapping;
  int64_t slot_map_stride;
  int64_t num_tokens;
  const float* boundaries[2];
  int32_t bits[2];
  const uint16_t* rot_hi;     // bf16 bit patterns [D][D], row-major (row j: output j)
  const uint16_t* rot_lo;
  unsigned int* err;
  int32_t box_h;              // heads per box (the tile is box_h x (128 / box_h) pairs)
  int32_t nst;                // input stages: 2 (the next tile's copies overlap) or 1
  uint32_t wait_ms;
  // test export: write u = y / n and n of the K rows instead of storing slots
  int32_t export_mode;
  float* u_out;
  int64_t u_stride;
  float* n_out;
};

// K and V inputs as (D, h_kv, tokens) bf16, boxes of (64, box_h, 128 / box_h), 128-byte
// swizzle.
struct DenseAppendMaps {
  CUtensorMap k, v;
};

constexpr int kDenseRows = 128;      // pairs per tile (the MMA's M)
constexpr int kDenseThreads = 512;   // 16 warps: (row quarter, kind, column half)

// ---------------------------------------------------------------------------
// tcgen05 / tensor memory wrappers (cta_group::1, no multicast)
// ---------------------------------------------------------------------------

// Shared-memory matrix descriptor of a K-major operand with the 128-byte swizzle:
// start address >> 4 in bits 0-13, leading byte offset (unused by this layout, 16 B) in
// bits 16-29, stride byte offset 1024 (between 8-row groups) in bits 32-45, descriptor
// version 1 in bits 46-47, base offset 0, layout type 2 (SWIZZLE_128B) in bits 61-63.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}

// Instruction descriptor of kind::f16 with bf16 A and B (both K-major), fp32 accumulate,
// M = 128, N = n.
__host__ __device__ constexpr uint32_t dense_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The mbarrier receives one arrival once all earlier tcgen05 operations of this thread
// are complete.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
// 32 consecutive fp32 columns of this thread's tensor-memory lane (warp quarter).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// Byte offset of element (row, col) of a [rows][D] bf16 operand stored as 64-column
// blocks of `rows` x 128 bytes with the 128-byte swizzle.
__host__ __device__ __forceinline__ uint32_t sw128_offset(int row, int col, int rows) {
  const int blk = col >> 6, c = col & 63;
  return (uint32_t)(blk * rows * 128 + row * 128 + ((((c >> 3) ^ (row & 7)) & 7) << 4) +
                    (c & 7) * 2);
}

// Encode 32 unit coordinates and pack their codes LSB-first into BITS words (32 codes
// of BITS bits fill exactly BITS words).  Same decision as encode_pack: the bucket
// table and one compare when FAST, else the Eytzinger search.
template <int BITS, bool FAST>
__device__ __forceinline__ void encode32(const float (&u)[32], const EncodeTables* t,
                                         uint32_t* words) {
  uint32_t acc[BITS];
#pragma unroll
  for (int w = 0; w < BITS; ++w) acc[w] = 0u;
  const uint32_t bnd_win = smem_u32(t->bnd);
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int bit = j * BITS;
    const int w0 = bit >> 5, o0 = bit & 31;
    uint32_t code;
    if constexpr (FAST) {
      const uint32_t k4 = t->k4[__float_as_uint(u[j]) >> kBucketShift];
      code = (k4 >> 2) + (u[j] > lds_f32(bnd_win | k4) ? 1u : 0u);
    } else {
      int e = 1;
#pragma unroll
      for (int st = 0; st < BITS; ++st) e = 2 * e + (u[j] > t->eytz[e - 1] ? 1 : 0);
      code = (uint32_t)(e - (1 << BITS));
    }
    acc[w0] += code << o0;
    if (o0 + BITS > 32) acc[w0 + 1] += code >> (32 - o0);
  }
#pragma unroll
  for (int w = 0; w < BITS; ++w) words[w] = acc[w];
}

template <int BITS>
__device__ __forceinline__ void encode32_any(const float (&u)[32], const EncodeTables* t,
                                             int fast, uint32_t* words) {
  if constexpr (BITS <= 4) {
    if (fast) {
      encode32<BITS, true>(u, t, words);
      return;
    }
  }
  encode32<BITS, false>(u, t, words);
}

__device__ __forceinline__ void encode32_bits(int bits, const float (&u)[32], const EncodeTables* t,
                                              int fast, uint32_t* words) {
  switch (bits) {
    case 1: encode32_any<1>(u, t, fast, words); break;
    case 2: encode32_any<2>(u, t, fast, words); break;
    case 3: encode32_any<3>(u, t, fast, words); break;
    case 4: encode32_any<4>(u, t, fast, words); break;
    case 5: encode32_any<5>(u, t, fast, words); break;
    case 6: encode32_any<6>(u, t, fast, words); break;
    case 7: encode32_any<7>(u, t, fast, words); break;
    default: encode32_any<8>(u, t, fast, words); break;
  }
}

// Rare path of the epilogue: the row's y = R (x 2^-e) on the CUDA cores (fp32 fused
// multiply-add over k = 0 .. D-1, R = hi + lo read from the tables in global memory),
// for rows whose squares leave the range where the tensor-core product is exact to
// fp32 rounding.  Writes y[c * 32 .. c * 32 + 31].
template <int D>
__device__ __forceinline__ void dense_row_fallback(const DenseAppendParams& p,
                                                   const uint8_t* xrow_blk, int row, float s1,
                                                   float s2, int c, float (&y)[32]) {
#pragma unroll
  for (int jj = 0; jj < 32; ++jj) {
    const int j = c * 32 + jj;
    float acc = 0.f;
#pragma unroll 1
    for (int k = 0; k < D; ++k) {
      const uint16_t xb = *(const uint16_t*)(xrow_blk + sw128_offset(row, k, kDenseRows));
      const float x = __fmul_rn(__fmul_rn(bf16_bits_to_f32(xb), s1), s2);
      const float r = __fadd_rn(bf16_bits_to_f32(p.rot_hi[j * D + k]),
                                bf16_bits_to_f32(p.rot_lo[j * D + k]));
      acc = fmaf(r, x, acc);
    }
    y[jj] = acc;
  }
}

template <int D>
struct DenseSmem {
  static constexpr int ROT = D * D * 2;                 // one of R hi, R lo
  static constexpr int KIND = kDenseRows * D * 2;       // one kind's rows of a tile
  static constexpr int STAGE = 2 * KIND;                // K and V rows
  static constexpr int TABLES = 2 * (int)sizeof(EncodeTables);
  static __host__ __device__ constexpr int slot_words(int kbits, int vbits) {
    return (D * kbits / 8 + 4 + D * vbits / 8 + 4) / 4;
  }
  // words of the slot area: the tile's slots, and at least the norm pass's half-row
  // exchange ([2][2][128] u32 pairs)
  static __host__ __device__ constexpr int slot_area_words(int kbits, int vbits) {
    return kDenseRows * slot_words(kbits, vbits) > 2 * 2 * kDenseRows * 2
               ? kDenseRows * slot_words(kbits, vbits)
               : 2 * 2 * kDenseRows * 2;
  }
  // [R hi | R lo | nst stages] (1024-aligned), tables, slots, slot offsets, misc
  static __host__ __device__ constexpr int bytes(int kbits, int vbits, int nst) {
    return 1024 + 2 * ROT + nst * STAGE + TABLES + slot_area_words(kbits, vbits) * 4 +
           kDenseRows * 8 + 64;
  }
};

template <int D>
__global__ void __launch_bounds__(kDenseThreads, 1)
append_dense_kernel(DenseAppendParams p, const __grid_constant__ DenseAppendMaps maps) {
  using SM = DenseSmem<D>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* rot_s = smem;                                   // [hi | lo]
  uint8_t* stage_s = smem + 2 * SM::ROT;                   // [nst][K rows | V rows]
  EncodeTables* tabs = (EncodeTables*)(stage_s + p.nst * SM::STAGE);
  const int swords = SM::slot_words(p.bits[0], p.bits[1]);
  uint32_t* slots_s = (uint32_t*)((uint8_t*)tabs + SM::TABLES);   // [128][swords]
  int64_t* dst_s = (int64_t*)(slots_s + SM::slot_area_words(p.export_mode ? 1 : p.bits[0],
                                                              p.export_mode ? 1 : p.bits[1]));
  uint64_t* bars = (uint64_t*)(dst_s + kDenseRows);        // full[2], mma_done[2]
  uint32_t* tmem_slot = (uint32_t*)(bars + 4);
  int* flags = (int*)(tmem_slot + 1);                       // fast[2], dead
  // half-row sums of squares and maxima [kind][half][row] (ss, max |x| bits), in the slot
  // area while it is free (the norm pass, before the epilogue writes the slots)
  uint2* half_norm = (uint2*)slots_s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kind = (warp >> 2) & 1;                        // epilogue kind of this warp
  const int half = warp >> 3;                               // its half of the columns
  const int row = ((warp & 3) << 5) | lane;                 // epilogue row (TMEM lane)
  const int kwords = (D * p.bits[0] + 7) / 8 / 4 + 1;
  const int64_t npairs = p.num_tokens * p.h_kv;
  const int64_t ntiles = (npairs + kDenseRows - 1) / kDenseRows;
  // Two input stages and, where tensor memory holds two sets of accumulators (4 D <= 512
  // columns), a pipelined loop: the next tile's MMAs run while this tile's epilogue does.
  const bool pipe = p.nst == 2 && 4 * D <= 512;
  const uint32_t ncols = pipe ? 4 * D : 2 * D;              // K and V accumulators (x2)

  // rotation into shared memory (16-byte pieces: 8 consecutive k of one row j)
  for (int i = tid; i < 2 * D * D / 8; i += blockDim.x) {
    const int part = i / (D * D / 8), e = (i % (D * D / 8)) * 8;
    const int j = e / D, k = e % D;
    const uint4 v = *(const uint4*)((part ? p.rot_lo : p.rot_hi) + e);
    *(uint4*)(rot_s + part * SM::ROT + sw128_offset(j, k, D)) = v;
  }
  if (!p.export_mode) {                 // the export writes u: no tables
    build_tables(&tabs[0], p.boundaries[0], p.bits[0], tid, blockDim.x, &flags[0]);
    build_tables(&tabs[1], p.boundaries[1], p.bits[1], tid, blockDim.x, &flags[1]);
  }
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init(&bars[2], 1);
    mbar_init(&bars[3], 1);
    flags[2] = 0;
    fence_mbar_init();
  }
  fence_proxy_async_smem();         // the rotation is read by the tensor cores
  if (warp == 0) tmem_alloc(tmem_slot, ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (!p.export_mode) {
    build_bucket_table(&tabs[0], p.bits[0], tid, blockDim.x);
    build_bucket_table(&tabs[1], p.bits[1], tid, blockDim.x);
  }

  // tensor copies of tile `tile` (both kinds) into stage b, completing on bars[b]
  auto load_tile = [&](int64_t tile, int b) {
    const int64_t r0 = tile * kDenseRows;
    const int t0 = (int)(r0 / p.h_kv), h0 = (int)(r0 % p.h_kv);
    mbar_arrive_expect_tx(&bars[b], SM::STAGE);
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int blk = 0; blk < D / 64; ++blk)
        tensor_g2s_3d(stage_s + b * SM::STAGE + k * SM::KIND + blk * kDenseRows * 128,
                      k ? &maps.v : &maps.k, 64 * blk, h0, t0, &bars[b]);
  };
  // the MMAs of the tile staged in stage b into accumulator set a (tensor memory columns
  // [a 2D, a 2D + 2D)), committed to mma_done[a] (thread 0)
  auto issue_mma = [&](int b, int a) {
    const uint8_t* st = stage_s + b * SM::STAGE;
    const uint32_t idesc = dense_idesc(D);
#pragma unroll 1
    for (int k = 0; k < (p.export_mode ? 1 : 2); ++k) {
      const uint32_t a0 = smem_u32(st + k * SM::KIND);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t aoff = (ks >> 2) * (kDenseRows * 128) + (ks & 3) * 32;
        const uint32_t boff = (ks >> 2) * (D * 128) + (ks & 3) * 32;
#pragma unroll
        for (int part = 0; part < 2; ++part)
          umma_bf16(tmem + (uint32_t)(a * 2 * D + k * D), sw128_desc(a0 + aoff),
                    sw128_desc(smem_u32(rot_s + part * SM::ROT) + boff), idesc,
                    (ks > 0 || part > 0) ? 1u : 0u);
      }
    }
    umma_commit(&bars[2 + a]);
  };
  // slot offsets of the tile's pairs (threads 0 .. 127)
  auto slot_offsets = [&](int64_t r0, int nr) {
    if (tid < kDenseRows) {
      int64_t off = -1;
      if (tid < nr && !p.export_mode) {
        const int64_t pr = r0 + tid;
        const int64_t t = pr / p.h_kv, h = pr - t * p.h_kv;
        const int64_t slot = p.slot_mapping[t * p.slot_map_stride];
        if (slot >= 0) {
          if (slot < p.num_slots) {
            const int64_t blk = p.bs_shift >= 0 ? slot >> p.bs_shift : slot / p.block_size;
            const int64_t rr = slot - blk * p.block_size;
            off = blk * p.blk_stride + rr * p.row_stride + h * p.head_stride;
          } else {
            report_error(p.err, TQ_DEVERR_SLOT_RANGE);
          }
        }
      }
      dst_s[tid] = off;
    }
  };
  // Per-thread row state of the tile's norm pass.
  struct RowNorm {
    float ss, n, r, norm;
    uint32_t mx;
    int e;
    bool bad, in_range;
  };
  const bool active = !(p.export_mode && kind == 1);
  // the row's norm from the staged input (plain fp32 sum of squares in k order)
  auto norm_pass = [&](const uint8_t* xblk) -> RowNorm {
    RowNorm q;
    q.ss = 0.f;
    q.mx = 0u;
    if (active) {
#pragma unroll 4
      for (int c = half * (D / 16); c < (half + 1) * (D / 16); ++c) {
        const uint4 v = *(const uint4*)(xblk + sw128_offset(row, 8 * c, kDenseRows));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float lo = bf16_bits_to_f32(w[i] & 0xffffu), hi = __uint_as_float(w[i] & 0xffff0000u);
          q.ss = fmaf(lo, lo, q.ss);
          q.ss = fmaf(hi, hi, q.ss);
          q.mx = max(q.mx, max((w[i] << 16) & 0x7fffffffu, w[i] & 0x7fff0000u));
        }
      }
    }
    // the row's two halves (this thread's and the one of warp ^ 8): half 0's sum comes first
    half_norm[(kind * 2 + half) * kDenseRows + row] = make_uint2(__float_as_uint(q.ss), q.mx);
    __syncthreads();
    const uint2 o = half_norm[(kind * 2 + (half ^ 1)) * kDenseRows + row];
    __syncthreads();                    // the slot area is written by the epilogue next
    q.ss = half ? __fadd_rn(__uint_as_float(o.x), q.ss) : __fadd_rn(q.ss, __uint_as_float(o.x));
    q.mx = max(q.mx, o.y);
    q.bad = q.mx >= 0x7f800000u;
    q.in_range = q.ss >= 0x1p-60f && q.ss <= 0x1p100f;
    q.e = 0;
    q.n = sqrtf(q.ss);
    if (active && !q.in_range && !q.bad && q.mx != 0u) {
      // scaled sum of squares: the largest magnitude brought into [1, 2) (exact)
      q.e = exponent_of(q.mx);
      const float s1 = pow2f(-q.e / 2), s2 = pow2f(-q.e - (-q.e / 2));
      float ss2 = 0.f;
      for (int k = 0; k < D; ++k) {
        const float x = __fmul_rn(
            __fmul_rn(bf16_bits_to_f32(*(const uint16_t*)(xblk + sw128_offset(row, k, kDenseRows))),
                      s1),
            s2);
        ss2 = fmaf(x, x, ss2);
      }
      q.n = sqrtf(ss2);
    }
    q.r = q.n > 0.f ? __frcp_rn(q.n) : 0.f;
    q.norm = q.e == 0 ? q.n : __fmul_rn(__fmul_rn(q.n, pow2f(q.e / 2)), pow2f(q.e - q.e / 2));
    return q;
  };
  // epilogue of the tile (staged rows xblk, accumulator set a): u = y r, encode and pack
  // into the slots in shared memory (or, in export mode, write u and n)
  auto epilogue = [&](const uint8_t* xblk, int a, int64_t r0, int nr, const RowNorm& q) {
    const int bits = p.bits[kind];
    const int rwords = kind ? swords - kwords : kwords;
    uint32_t* orow = slots_s + row * swords + (kind ? kwords : 0);
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(a * 2 * D + kind * D);
#pragma unroll 1
    for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
      float y[32];
      tmem_ld32(tl + 32 * c, y);             // every thread of the warp takes part
      if (active && !q.in_range && !q.bad && q.mx != 0u) {
        const float s1 = pow2f(-q.e / 2), s2 = pow2f(-q.e - (-q.e / 2));
        dense_row_fallback<D>(p, xblk, row, s1, s2, c, y);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) y[i] = __fmul_rn(y[i], q.r);
      if (!active) continue;
      if (p.export_mode) {
        if (row < nr) {
          float* u = p.u_out + (r0 + row) * p.u_stride + 32 * c;
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = q.bad ? 0.f : y[i];
        }
      } else if (!q.bad) {
        encode32_bits(bits, y, &tabs[kind], flags[kind], orow + c * bits);
      } else {
        for (int w = 0; w < bits; ++w) orow[c * bits + w] = 0u;
      }
    }
    if (active && half == 0) {
      if (p.export_mode) {
        if (row < nr) p.n_out[r0 + row] = q.bad ? __uint_as_float(0x7FC00000u) : q.norm;
      } else {
        orow[rwords - 1] = q.bad ? 0x7FC00000u : __float_as_uint(q.norm);
        if (q.bad && row < nr) report_error(p.err, TQ_DEVERR_NONFINITE);
      }
    }
  };
  // the tile's slots to the page pool (lanes over (slot, word))
  auto store_slots = [&](int nr) {
    if (!p.export_mode) {
      for (int i = tid; i < nr * swords; i += blockDim.x) {
        const int rr = i / swords, w = i - rr * swords;
        const int64_t off = dst_s[rr];
        if (off >= 0) ((uint32_t*)(p.pages + off))[w] = slots_s[rr * swords + w];
      }
    }
  };
  auto fail = [&]() {
    report_error(p.err, TQ_DEVERR_TIMEOUT);
    flags[2] = 1;
  };
  const int64_t first = blockIdx.x;
  const int nst = p.nst;
  // operations issued by thread 0 and not yet waited for: copies into stage b (pend_full[b]
  // = completion parity, or -1) and MMAs into accumulator set a (pend_mma[a])
  int pend_full[2] = {-1, -1}, pend_mma[2] = {-1, -1};

  if (pipe) {
    // prologue: copies of the first two tiles, the MMAs of the first
    if (tid == 0 && first < ntiles) {
      load_tile(first, 0);
      pend_full[0] = 0;
      if (first + gridDim.x < ntiles) {
        load_tile(first + gridDim.x, 1);
        pend_full[1] = 0;
      }
      if (!mbar_wait(&bars[0], 0, p.wait_ms)) {
        fail();
      } else {
        pend_full[0] = -1;
        tc_fence_after();
        issue_mma(0, 0);
        pend_mma[0] = 0;
      }
    }
    __syncthreads();
    uint32_t it = 0;
    for (int64_t tile = first; tile < ntiles && !flags[2]; tile += gridDim.x, ++it) {
      const int b = (int)(it & 1u);                 // stage and accumulator set of the tile
      const uint32_t ph = (it >> 1) & 1u;           // their completion parity
      const int64_t r0 = tile * kDenseRows;
      const int nr = (int)imin64(kDenseRows, npairs - r0);
      const uint8_t* xblk = stage_s + b * SM::STAGE + kind * SM::KIND;
      slot_offsets(r0, nr);
      // the staged rows (thread 0 waited for them before the MMAs)
      if (tid != 0 && !mbar_wait(&bars[b], ph, p.wait_ms)) fail();
      const RowNorm q = norm_pass(xblk);
      // the next tile's MMAs into the other accumulator set, overlapping this epilogue
      // (its rows were requested one tile ago; the set was released at the last barrier)
      if (tid == 0 && tile + gridDim.x < ntiles && !flags[2]) {
        const uint32_t nph = ((it + 1) >> 1) & 1u;
        if (!mbar_wait(&bars[b ^ 1], nph, p.wait_ms)) {
          fail();
        } else {
          pend_full[b ^ 1] = -1;
          tc_fence_after();
          issue_mma(b ^ 1, b ^ 1);
          pend_mma[b ^ 1] = (int)nph;
        }
      }
      __syncwarp();
      // this tile's accumulators (every thread waits; a launch that stopped never
      // completes them)
      if (!mbar_wait(&bars[2 + b], ph, p.wait_ms)) {
        if (tid == 0) report_error(p.err, TQ_DEVERR_TIMEOUT);
        flags[2] = 1;
      } else if (tid == 0) {
        pend_mma[b] = -1;
      }
      __syncwarp();
      tc_fence_after();
      epilogue(xblk, b, r0, nr, q);
      // tensor memory set b, stage b and the slots are complete
      tc_fence_before();
      __syncthreads();
      store_slots(nr);
      __syncthreads();
      // stage b is free: the rows of the tile after next come in
      if (tid == 0 && !flags[2] && tile + 2 * (int64_t)gridDim.x < ntiles) {
        load_tile(tile + 2 * (int64_t)gridDim.x, b);
        pend_full[b] = (int)(((it + 2) >> 1) & 1u);
      }
    }
  } else {
    if (tid == 0 && first < ntiles) {
      load_tile(first, 0);
      pend_full[0] = 0;
    }
    __syncthreads();
    uint32_t it = 0;
    for (int64_t tile = first; tile < ntiles; tile += gridDim.x, ++it) {
      const int b = nst == 2 ? (int)(it & 1) : 0;
      const uint32_t full_parity = nst == 2 ? (it >> 1) & 1u : it & 1u;
      const int64_t r0 = tile * kDenseRows;
      const int nr = (int)imin64(kDenseRows, npairs - r0);
      if (tid == 0) {
        // the MMAs of this tile once its rows have landed
        if (!mbar_wait(&bars[b], full_parity, p.wait_ms)) {
          fail();
        } else {
          pend_full[b] = -1;
          tc_fence_after();
          issue_mma(b, 0);
          pend_mma[0] = (int)(it & 1u);
          // with two stages the next tile's rows come in meanwhile (its stage was freed at
          // the end of the previous tile)
          if (nst == 2 && tile + gridDim.x < ntiles) {
            load_tile(tile + gridDim.x, b ^ 1);
            pend_full[b ^ 1] = (int)(((it + 1) >> 1) & 1u);
          }
        }
      }
      __syncwarp();
      slot_offsets(r0, nr);
      // the staged rows are read below: every thread waits for the tile's copies (thread 0
      // has already waited for them before issuing the MMAs)
      if (tid != 0 && !mbar_wait(&bars[b], full_parity, p.wait_ms)) fail();
      const uint8_t* xblk = stage_s + b * SM::STAGE + kind * SM::KIND;
      const RowNorm q = norm_pass(xblk);
      // the accumulators (every thread waits; a launch that stopped never completes them)
      if (!mbar_wait(&bars[2], it & 1u, p.wait_ms)) {
        if (tid == 0) report_error(p.err, TQ_DEVERR_TIMEOUT);
        flags[2] = 1;
      } else if (tid == 0) {
        pend_mma[0] = -1;
      }
      __syncwarp();
      tc_fence_after();
      epilogue(xblk, 0, r0, nr, q);
      // tensor memory, the stage and the slots are complete
      tc_fence_before();
      __syncthreads();
      store_slots(nr);
      __syncthreads();
      if (flags[2]) break;
      // with one stage the next tile's rows come in now that the stage is free
      if (nst == 1 && tid == 0 && tile + gridDim.x < ntiles) {
        load_tile(tile + gridDim.x, 0);
        pend_full[0] = (int)((it + 1) & 1u);
      }
    }
  }
  // copies and MMAs still in flight (a launch that stopped early) complete before the
  // tensor memory is released and the CTA ends (bounded waits)
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      if (pend_full[b] >= 0) mbar_wait(&bars[b], (uint32_t)pend_full[b], p.wait_ms);
      if (pend_mma[b] >= 0) mbar_wait(&bars[2 + b], (uint32_t)pend_mma[b], p.wait_ms);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, ncols);
}

}  // namespace tq
