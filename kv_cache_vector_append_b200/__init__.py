"""B200-native TurboQuant packed-KV quantize-append and paged decode.

Thin Python binding over the C ABI of ``libtq.so`` (declared in
``include/tq.h``).  Every step of the hot path runs in the library's CUDA
kernels; this module only marshals torch tensors into ``tq_tensor`` views and
checks status codes.  There is no CPU fallback: if the library is missing or a
call fails, an exception is raised.

Public API (names follow the C entry points):
    slot_bytes(D, k_bits, v_bits) -> int
    load_codebooks(D, k_bits, v_bits, device) -> Codebooks
    quantize_append(pages, slot_mapping, k, v, codebooks, sign_seed, stream=None)
    paged_decode(out, q, pages, block_table, seq_lens, codebooks, sign_seed, scale, stream=None)
    paged_decode_hot(out, q, pages, block_table, seq_lens, hot_k, hot_v, hot_lens, ...)
                                # same, plus an uncompressed hot window (sinks, recent tokens)
    quantize_append_qjl(...), paged_decode_qjl(...), slot_bytes_qjl(D, kb, vb)
                                # keys with the QJL residual sketch
    paged_decode_noalloc(...)   # same, with the library's fixed scratch (no allocation)
    rotate_unit(u, norm, x, sign_seed, stream=None)       # test export of the rotation
    load_rotation(D, device) -> Rotation                  # dense (QR) rotation table
    quantize_append_dense(pages, slot_mapping, k, v, codebooks, rotation, stream=None)
    paged_decode_dense(out, q, pages, block_table, seq_lens, codebooks, rotation, scale, ...)
    rotate_unit_dense(u, norm, x, rotation, stream=None)  # test export of the dense rotation
    decode_workspace_size(...), set_workspace(tensor), get_device_error(stream=None)
"""

from ._binding import (  # noqa: F401
    Codebooks,
    TQError,
    DEVERR_BLOCK_RANGE,
    DEVERR_NONFINITE,
    DEVERR_SEQLEN_RANGE,
    DEVERR_SLOT_RANGE,
    DEVERR_TIMEOUT,
    debug_inject_merge_stall,
    decode_workspace_size,
    get_device_error,
    library_path,
    load_codebook_table,
    load_codebooks,
    load_rotation,
    Rotation,
    quantize_append_dense,
    paged_decode_dense,
    rotate_unit_dense,
    paged_decode,
    paged_decode_hot,
    paged_decode_qjl,
    quantize_append_qjl,
    slot_bytes_qjl,
    paged_decode_noalloc,
    quantize_append,
    rotate_unit,
    set_workspace,
    slot_bytes,
    version,
)
