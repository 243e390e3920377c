/*
 * tq.h -- C ABI of the B200 TurboQuant packed-KV library (libtq.so).
 *
 * Two operations make up the hot path:
 *
 *   tq_quantize_append  rotate each K/V row with a randomized Hadamard transform,
 *                       store its fp32 L2 norm, Lloyd-Max-encode every rotated unit
 *                       coordinate and bit-pack the codes into the row's page slot;
 *   tq_paged_decode     one attention decode step straight over the packed pages:
 *                       rotate q once, score each key on its codes, online softmax,
 *                       accumulate V in the rotated domain, inverse-rotate the output.
 *
 * Sources (page title, section):
 *   TorbuQuant (ginkgoq.github.io/TurboQuant), "TQ4 page tensor" diagram -- page
 *     tensor [num_blocks, block_size, num_kv_heads, slot_bytes], slot -> (block, row),
 *     slot = [K: packed indices, fp32 norm][V: packed indices, fp32 norm],
 *     K bytes ceil(D*k_bits/8)+4, V bytes ceil(D*v_bits/8)+4, optional padding;
 *     the stages "Quantize: rotate, normalize, codebook-encode, pack" and "Store".
 *   tq-kv (shadowgraph.io), "How It Works" step 3 (randomized Hadamard transform)
 *     and "Library API" (generate_signs(dim, seed), pre_rotate_query_with_signs,
 *     fused_attention_scores on compressed keys); "Custom CUDA Kernel Stack"
 *     (flash decode with split-KV and online softmax; attention score without
 *     decompression).
 *   turboquant_serve 0.1.2, "Architecture" (update(): rotate, normalize,
 *     Lloyd-Max encode, bit-pack; _decode(): unpack, decode, restore magnitude,
 *     rotate back; one rotation per head_dim; codebooks fitted once and shared).
 *   turboquant_pro 1.4.2, "How It Works" (norm preserved alongside the bits;
 *     8 x 3-bit = 3 bytes) and "Fused CUDA decode" (split-K decode on the codes).
 *
 * Conventions where the pages are silent (the library and its tests agree on them):
 *   - signs: s_j = -1 if bit 63 of the j-th SplitMix64 output seeded with
 *     sign_seed is set, else +1 (j = 0..D-1); the same signs serve K, V, q and
 *     every head; rotation y = (1/sqrt(D)) H (s * x), H the natural-order
 *     (Sylvester) Hadamard matrix;
 *   - norm: L2 norm of the input row, stored as fp32 (rows of any finite magnitude;
 *     a norm beyond the fp32 range stores +inf); unit coordinates u = y / n;
 *   - code: idx = number of boundaries b_i with b_i < u (ties to the lower cell);
 *     a zero row stores norm 0 and codes idx(0); a row holding a non-finite value
 *     stores codes 0 and a quiet-NaN norm (0x7FC00000) and raises
 *     TQ_DEVERR_NONFINITE;
 *   - packing: code j fills bits [j*bits, (j+1)*bits) of a little-endian bit
 *     stream (bit p = bit p%8 of byte p/8); the fp32 norm follows, little endian;
 *   - GQA: query head h reads KV head h / (H_q / H_kv).
 *
 * Memory: every pointer below is a DEVICE pointer unless stated otherwise.  The
 * caller owns all buffers.  Calls are asynchronous on `stream` (a cudaStream_t
 * passed as void*, NULL = legacy default stream); host-side validation errors are
 * returned synchronously and nothing is enqueued.  Errors found by a kernel (an
 * out-of-range slot or block id, a non-finite input row) are OR-ed into a
 * per-device error word read by tq_get_device_error(); the offending row or
 * block is skipped, nothing faults.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,  /* bad pointer, shape, stride, dtype or parameter   */
  TQ_ERR_UNSUPPORTED = 2,  /* valid but not built: head_dim, bits or GQA group */
  TQ_ERR_CUDA = 3,         /* a CUDA runtime call failed (launch, memcpy, ...)  */
  TQ_ERR_DEVICE = 4,       /* a kernel reported an error (see the error word)  */
  TQ_ERR_WORKSPACE = 5     /* workspace missing or too small                    */
} tq_status;

typedef enum {
  TQ_U8 = 0,
  TQ_I32 = 1,
  TQ_I64 = 2,
  TQ_F32 = 3,
  TQ_BF16 = 4,
  TQ_F16 = 5
} tq_dtype;

/* Device error word bits (tq_get_device_error). */
#define TQ_DEVERR_SLOT_RANGE 0x1    /* slot_mapping entry >= num_blocks*block_size */
#define TQ_DEVERR_BLOCK_RANGE 0x2   /* block_table entry outside [0, num_blocks)   */
#define TQ_DEVERR_NONFINITE 0x4     /* a K/V input row held a NaN or an infinity   */
#define TQ_DEVERR_SEQLEN_RANGE 0x8  /* seq_len < 0 or > max_blocks*block_size      */
#define TQ_DEVERR_TIMEOUT 0x10      /* a bounded wait inside a kernel gave up        */
#define TQ_DEVERR_LAYOUT 0x20       /* the decode kernel's shared-memory layout did not
                                       match its launch; the launch did nothing      */

/* A strided view of a device array.  Strides are in ELEMENTS; shape[i] and
 * stride[i] for i >= ndim are ignored.  data must be aligned to the element size. */
typedef struct {
  void* data;
  int32_t dtype;      /* tq_dtype */
  int32_t ndim;
  int64_t shape[4];
  int64_t stride[4];
} tq_tensor;

/* One fp32 Lloyd-Max table (Beta-sphere density for `dim`): `centroids` holds
 * 2^bits ascending values, `boundaries` the 2^bits - 1 ascending cell edges.
 * Both are device pointers, 4-byte aligned, owned by the caller and read by
 * every launch ("fitted once ... and shared", turboquant_serve, "Codebook sharing"). */
typedef struct {
  int32_t dim;
  int32_t bits;
  const float* centroids;
  const float* boundaries;
} tq_codebook;

typedef struct {
  tq_codebook k;
  tq_codebook v;
} tq_codebooks;

/* The dense random rotation R (turboquant_serve 0.1.2, "Architecture" and "Rotation": a
 * fixed random orthogonal matrix, seeded by head_dim; TorbuQuant, "Current Status": QR
 * rotation) as two bf16 matrices: R = hi + lo, [dim][dim] row-major (row j gives output
 * coordinate j), bf16 bit patterns in device memory, 16-byte aligned, owned by the caller.
 * The library's data files rotations/qr_d<D>.tqrt hold them (hi = bf16 of the seeded
 * Haar matrix, lo = bf16 of the remainder; R is exact in fp32 and orthogonal to ~1e-5). */
typedef struct {
  int32_t dim;
  const uint16_t* hi;
  const uint16_t* lo;
} tq_rotation;

/* Bytes of one slot before padding: (ceil(D*k_bits/8)+4) + (ceil(D*v_bits/8)+4)
 * (TorbuQuant, "TQ4 page tensor").  Host only; *out receives the value.
 * Errors: TQ_ERR_INVALID_ARG for dim < 1, bits outside 1..8 or out == NULL. */
TQ_API tq_status tq_slot_bytes(int32_t dim, int32_t k_bits, int32_t v_bits, int32_t* out);

/* Quantize-append (TorbuQuant "Quantize" and "Store"; turboquant_serve update()).
 *
 *   pages        u8  [num_blocks, block_size, H_kv, slot_stride]; the last dim is
 *                contiguous, slot_stride >= tq_slot_bytes(D, k_bits, v_bits) and a
 *                multiple of 8; bytes beyond slot_bytes are never written.
 *   slot_mapping i64 [T]: token t goes to slot s = slot_mapping[t], i.e.
 *                page[s / block_size, s % block_size, h, :] for every KV head h;
 *                s < 0 skips the token; s >= num_blocks*block_size skips it and
 *                raises TQ_DEVERR_SLOT_RANGE.
 *   k, v         [T, H_kv, D] in bf16, f16 or f32 (same dtype); the last dim is
 *                contiguous; rows are read exactly (converted to fp32).
 *   cb           host pointer to the K and V tables (device arrays inside);
 *                cb->k.dim == cb->v.dim == D, cb->k.bits == k_bits, cb->v.bits == v_bits.
 *   sign_seed    SplitMix64 seed of the rotation signs.
 *   k_bits, v_bits  1..8.  D must be 64, 128 or 256.
 * Two tokens mapped to the same slot race (either row may win).
 * Two launches: the fast path, then a redo that returns at once unless some row's sum
 * of squares left the fast path's range (rows of magnitude beyond about 1e14 or below
 * about 1e-10, zero rows, non-finite rows), in which case the whole call is done again
 * with an exact power-of-two rescaling of those rows.  The two share a per-device flag:
 * calls on one device whose kernels overlap on the GPU (unordered streams) must be
 * ordered.
 * Fast paths (same results, chosen per call on the host):
 *   - k and v are staged by tensor copies when they are 16-bit, 16-byte aligned with
 *     token and head strides that are multiples of 8 elements, and H_kv divides
 *     2048/D or is a multiple of it;
 *   - each token's slots are stored with one bulk copy when, in addition to that H_kv
 *     rule, slot_stride == tq_slot_bytes(...), pages is 16-byte aligned with block and
 *     row strides that are multiples of 16, and the token's run of slots is a
 *     multiple of 16 bytes;
 *   - otherwise, when pages is 16-byte aligned with block, row and head strides that
 *     are multiples of 16 (a padded slot_stride), each slot's first
 *     (slot_bytes & ~15) bytes are stored by one bulk copy and the rest by 4-byte
 *     stores; the padding is not written.
 *   Other layouts take lane-wise copies.
 * Errors: TQ_ERR_INVALID_ARG / TQ_ERR_UNSUPPORTED (nothing enqueued), TQ_ERR_CUDA. */
TQ_API tq_status tq_quantize_append(tq_tensor pages, tq_tensor slot_mapping, tq_tensor k,
                             tq_tensor v, const tq_codebooks* cb, uint64_t sign_seed,
                             int32_t k_bits, int32_t v_bits, void* stream);

/* Paged decode (tq-kv "Library API" fused scores on compressed keys; "Custom CUDA
 * Kernel Stack" flash decode v2 split-KV with online softmax; turboquant_pro
 * "Fused CUDA decode").
 *
 *   out          [B, H_q, D], f32 or the dtype of q; last dim contiguous.
 *                out[b, h] = sum_t softmax_t(scale * <q[b,h], k_hat_t>) v_hat_t over
 *                t < seq_lens[b], where k_hat/v_hat are the dequantized rows
 *                norm * R^T c[idx] of KV head h / (H_q/H_kv).  seq_lens[b] == 0 gives 0.
 *   q            [B, H_q, D] in bf16, f16 or f32; last dim contiguous.
 *   pages        as in tq_quantize_append (k_bits/v_bits taken from cb).
 *   block_table  i32 [B, max_blocks]: token t of sequence b lives in block
 *                block_table[b, t / block_size], row t % block_size.  Entries past
 *                the sequence are not read.  An entry outside [0, num_blocks) raises
 *                TQ_DEVERR_BLOCK_RANGE and its block is skipped.
 *   seq_lens     i32 [B]; 0 <= seq_lens[b] <= max_blocks * block_size, otherwise
 *                TQ_DEVERR_SEQLEN_RANGE and the sequence gives 0.
 *   scale        softmax scale (typically 1/sqrt(D)).
 * K and V code widths (cb->k.bits, cb->v.bits): each of 2, 3, 4 and 8, in any pair
 * (TQ_ERR_UNSUPPORTED otherwise; tq_quantize_append takes 1..8).
 * H_q must be a multiple of H_kv with H_q / H_kv <= 16; block_size must be 16;
 * B * H_q < 2^31.  H_kv is at most 16 (8 when D = 256 or H_q / H_kv > 8), and a staged block of all
 * KV heads plus the code tables must fit in shared memory: with 8-bit tables that
 * excludes 16 KV heads at D = 128 and 8 at D = 256 (TQ_ERR_UNSUPPORTED;
 * tq_decode_plan_probe tells in advance).
 * One cooperative kernel launch: the merge of a sequence's partial results waits
 * (bounded, about 2 s) until every CTA that covers the sequence has published its
 * part; the merge work is spread over all CTAs.  A wait that gives up raises
 * TQ_DEVERR_TIMEOUT, leaves the affected query heads' output unwritten, and still
 * returns the merge counters to zero, so the next call runs normally.
 * Uses the per-device workspace (tq_set_workspace, or allocated by the library on
 * the first call that needs more, and kept until process exit).
 * Errors: TQ_ERR_INVALID_ARG / TQ_ERR_UNSUPPORTED / TQ_ERR_WORKSPACE (nothing
 * enqueued), TQ_ERR_CUDA. */
TQ_API tq_status tq_paged_decode(tq_tensor out, tq_tensor q, tq_tensor pages,
                          tq_tensor block_table, tq_tensor seq_lens,
                          const tq_codebooks* cb, uint64_t sign_seed, float scale,
                          void* stream);

/* The QJL residual sketch of the keys (tq-kv, "How It Works" step [5]: SRHT QJL error
 * correction; TorbuQuant, "Current Status": QJL residual).  After the Lloyd-Max code,
 * each K row also stores the 1-bit sketch of its rotated-domain residual r = u - c[idx]:
 * z_j = [(S r)_j >= 0] with S = (1/sqrt(D)) H diag(s2), a second randomized Hadamard
 * transform whose signs s2 come from SplitMix64 seeded with qjl_seed, and the fp32
 * gamma = ||r||.  K region = [packed codes | fp32 norm | D sign bits, LSB-first | fp32
 * gamma]; the V region follows unchanged.  Slot bytes: tq_slot_bytes_qjl (the pages'
 * slot_stride is at least that and a multiple of 8, so it may need padding).
 * Supported: D = 128 or 256 (the append), K widths 2, 3, 4 (the decode).  Same
 * arguments, layouts and errors as tq_quantize_append / tq_paged_decode otherwise; a
 * non-finite K row stores z = 0 and gamma = 0. */
TQ_API tq_status tq_slot_bytes_qjl(int32_t dim, int32_t k_bits, int32_t v_bits, int32_t* out);
TQ_API tq_status tq_quantize_append_qjl(tq_tensor pages, tq_tensor slot_mapping, tq_tensor k,
                                        tq_tensor v, const tq_codebooks* cb, uint64_t sign_seed,
                                        uint64_t qjl_seed, int32_t k_bits, int32_t v_bits,
                                        void* stream);
/* Decode over slots written by tq_quantize_append_qjl: each key is scored with its QJL
 * correction, scale nK (<R q, c[idx]> + gamma sqrt(pi/2)/sqrt(D) <S R q, 2z - 1>), the
 * second term as one more mma per k-step on +-1 fragments built from the sign bits. */
TQ_API tq_status tq_paged_decode_qjl(tq_tensor out, tq_tensor q, tq_tensor pages,
                                     tq_tensor block_table, tq_tensor seq_lens,
                                     const tq_codebooks* cb, uint64_t sign_seed,
                                     uint64_t qjl_seed, float scale, void* stream);

/* Paged decode with an uncompressed hot window (turboquant_pro 1.4.2, "Fused CUDA
 * decode": the fp16 hot window is merged through the online softmax, and "Streaming
 * cache"; tq-kv, "How It Works", "3-Fix for GGUF Models": sink tokens stay FP16, the
 * current token is lossless).  Same as tq_paged_decode, except that sequence b also
 * attends to hot tokens 0 .. hot_lens[b]-1 of hot_k / hot_v, inside the same softmax:
 *   out[b, h] = sum_t softmax_t(scale * <q[b,h], key_t>) value_t over the seq_lens[b]
 *               packed tokens (dequantized) and the hot tokens (read exactly).
 *   hot_k, hot_v  [B, W, H_kv, D] in bf16, f16 or f32 (same dtype and strides); the
 *                 last dim contiguous.  The caller keeps there whichever tokens stay
 *                 uncompressed (the first few "sink" tokens, the most recent ones); their
 *                 positions do not enter the result.  A token should be in the pages or
 *                 in the window, not both.
 *   hot_lens      i32 [B]; an entry outside [0, W] raises TQ_DEVERR_SEQLEN_RANGE and
 *                 counts as 0.  A sequence with seq_lens[b] == 0 attends to its hot
 *                 tokens alone; with no tokens at all it gives 0.
 * The packed tokens are reduced as in tq_paged_decode; the CTA that finishes a query
 * head computes the hot tokens' partial (fp32) and joins the two partials with one
 * rescale before the division by the softmax sum.
 * Errors: as tq_paged_decode, plus TQ_ERR_INVALID_ARG for mismatched hot tensors. */
TQ_API tq_status tq_paged_decode_hot(tq_tensor out, tq_tensor q, tq_tensor pages,
                                     tq_tensor block_table, tq_tensor seq_lens,
                                     tq_tensor hot_k, tq_tensor hot_v, tq_tensor hot_lens,
                                     const tq_codebooks* cb, uint64_t sign_seed, float scale,
                                     void* stream);

/* Allocation-free variant of tq_paged_decode (this library's own addition; the
 * pages describe no counterpart).  Same arguments, semantics and results as
 * tq_paged_decode, but its scratch is a fixed device array inside the library
 * (TQ_NOALLOC_SCRATCH_BYTES bytes, held by every device that loads the library
 * until the process exits) instead of a workspace the caller sets or the library
 * allocates.  It is meant for callers that must not allocate device memory on
 * the call path: a serving loop that keeps every allocation out of its steady
 * state (cudaMalloc/cudaFree can synchronise the device and fragment a pooled
 * allocator), or an embedding runtime that owns all device memory and forbids
 * libraries from allocating behind its back.  It calls no cudaMalloc, cudaFree or
 * allocating library routine.
 *
 *   - The first call on each device looks up the array's device address on that
 *     device (cudaGetSymbolAddress, which may load the library's module there);
 *     make that first call outside any stream capture.
 *   - A geometry whose scratch would exceed TQ_NOALLOC_SCRATCH_BYTES (see
 *     tq_decode_workspace_size for the size) is rejected with TQ_ERR_WORKSPACE and
 *     nothing is enqueued.
 *   - Every call on a device shares the one array.  It starts zeroed and every
 *     call leaves its merge counters at zero again.  Calls whose kernels overlap on
 *     the GPU (different streams without ordering) race on it: order them. */
#define TQ_NOALLOC_SCRATCH_BYTES (16u << 20)
TQ_API tq_status tq_paged_decode_noalloc(tq_tensor out, tq_tensor q, tq_tensor pages,
                                         tq_tensor block_table, tq_tensor seq_lens,
                                         const tq_codebooks* cb, uint64_t sign_seed, float scale,
                                         void* stream);

/* Workspace bytes tq_paged_decode needs for this geometry (host only).  The
 * workspace holds 2 * batch u32 merge counters at its start (zero between calls:
 * each call clears the ones it raised) and the split-KV partial results (m, l, O')
 * in fp32. */
TQ_API tq_status tq_decode_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                   int32_t head_dim, int32_t max_blocks, int32_t block_size,
                                   size_t* bytes);

/* Give the library a caller-owned device workspace for the CURRENT device
 * (ptr 256-byte aligned; NULL releases the association).  The library zeroes it
 * here (cudaMemset, synchronous) and never frees it; the caller must not write to
 * it while it is set.  Calls that use one device's workspace must be ordered on the
 * GPU (one stream, or events); concurrent decodes on one device race on it. */
TQ_API tq_status tq_set_workspace(void* ptr, size_t bytes);

/* Read and clear the current device's error word (TQ_DEVERR_* bits).  Host
 * pointer `out`; synchronises `stream` first.  When the word is non-zero it also
 * clears the merge counters of the device's workspaces, which a failed decode may
 * have left raised. */
TQ_API tq_status tq_get_device_error(int32_t* out, void* stream);

/* Test export of the rotation used by tq_quantize_append: for each row x of
 * `x` [N, D] (bf16/f16/f32), writes u = y / n with y = (1/sqrt(D)) H (s*x), n = ||x||,
 * in fp32 to `u` [N, D] and fp32(n) to `norm` [N], computed with exactly the
 * device arithmetic the append kernel uses (so encoding these u on the host
 * reproduces the kernel's codes bit for bit). */
TQ_API tq_status tq_rotate_unit(tq_tensor u, tq_tensor norm, tq_tensor x, uint64_t sign_seed,
                         void* stream);

/* Quantize-append with the dense rotation (turboquant_serve 0.1.2, "Architecture":
 * rotate k, v = k @ R, then normalize, encode and pack; turboquant_pro 1.4.2, "Fused CUDA
 * decode": rotation and quantization in one tiled GEMM).  Same slot layout, norm,
 * encode and errors as tq_quantize_append, with y = R x in place of the randomized
 * Hadamard transform: u = y / ||x||.  y is one tcgen05 GEMM per tile of 128 (token, head)
 * rows (bf16 x bf16 -> fp32 in tensor memory, R as hi and lo).
 *   rot   host pointer; rot->dim == D.
 * Supported: D = 64 or 128; k, v bf16, 16-byte aligned with token and head strides that
 * are multiples of 8 elements; H_kv a divisor or a multiple of 128 (TQ_ERR_UNSUPPORTED
 * otherwise).  Rows whose sum of squares leaves [2^-60, 2^100] are rotated on the CUDA
 * cores after an exact power-of-two rescaling. */
TQ_API tq_status tq_quantize_append_dense(tq_tensor pages, tq_tensor slot_mapping, tq_tensor k,
                                          tq_tensor v, const tq_codebooks* cb,
                                          const tq_rotation* rot, int32_t k_bits, int32_t v_bits,
                                          void* stream);

/* Paged decode with the dense rotation: as tq_paged_decode (sign_seed unused), with
 * q' = R q and o = R^T O' / l (fp32 on the CUDA cores, once per query head). */
TQ_API tq_status tq_paged_decode_dense(tq_tensor out, tq_tensor q, tq_tensor pages,
                                       tq_tensor block_table, tq_tensor seq_lens,
                                       const tq_codebooks* cb, const tq_rotation* rot, float scale,
                                       void* stream);

/* Test export of the dense append's rotation: for each bf16 row x of `x` [N, D] writes
 * u = R x / ||x|| (fp32, [N, D], unit stride) and fp32(||x||) to `norm` [N] with exactly
 * the arithmetic of tq_quantize_append_dense (the same kernel), so that encoding these u
 * on the host reproduces its codes bit for bit.  Same limits as that call. */
TQ_API tq_status tq_rotate_unit_dense(tq_tensor u, tq_tensor norm, tq_tensor x,
                                      const tq_rotation* rot, void* stream);

/* Test export for failure detection without a GPU fault (this library's own addition;
 * the pages describe no counterpart).  The NEXT decode launch on the current device
 * (tq_paged_decode or tq_paged_decode_noalloc) bounds its waits by `wait_ms`
 * milliseconds instead of about 2 s, and its CTA number `withhold_cta` never announces
 * its partial results.  So the CTAs that share a sequence with it give up waiting, raise
 * TQ_DEVERR_TIMEOUT, and write no output for that sequence (a withheld CTA past the
 * grid changes nothing).  One shot: later launches are normal.  Host only; nothing is
 * enqueued.
 * Errors: TQ_ERR_INVALID_ARG for withhold_cta < 0 or wait_ms outside 1..2000. */
TQ_API tq_status tq_debug_inject_merge_stall(int32_t withhold_cta, int32_t wait_ms);

/* Test export of the decode kernel's shared-memory plan for one call geometry on a
 * device described by num_sms, max_smem_optin (bytes one CTA may use) and
 * dyn_smem_base (the shared-window address where dynamic shared memory starts).
 * Host only: no device call.  out[14] receives, in order: wph, nst, row_pitch,
 * stage_bytes, lut_win, lut_off, lut_bytes, stage_lo_off, stage_hi_off, n_low,
 * misc_off, smem bytes, copy_mode (1: 2-D tensor box, 0: 1-D bulk copy), warps per CTA.
 * Errors: TQ_ERR_INVALID_ARG for out == NULL or non-positive sizes; TQ_ERR_UNSUPPORTED
 * when no layout fits. */
TQ_API tq_status tq_decode_plan_probe(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                      int32_t head_dim, int32_t k_bits, int32_t v_bits,
                                      int32_t slot_stride, int32_t max_blocks, int32_t num_sms,
                                      int32_t max_smem_optin, uint32_t dyn_smem_base,
                                      int64_t* out);

/* Static description of a status code (never NULL). */
TQ_API const char* tq_status_string(tq_status status);

/* Library version, e.g. "0.1.0". */
TQ_API const char* tq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
