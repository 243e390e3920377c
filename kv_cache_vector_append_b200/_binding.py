"""ctypes binding of libtq.so: tensor marshalling and status checks only."""

from __future__ import annotations

import ctypes
import os
import struct
from dataclasses import dataclass

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libtq.so")
_CODEBOOK_DIR = os.path.join(_PKG, "codebooks")

# tq_status
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_DEVICE, ERR_WORKSPACE = range(6)
# tq_dtype
U8, I32, I64, F32, BF16, F16 = range(6)
# device error word bits
DEVERR_SLOT_RANGE = 0x1
DEVERR_BLOCK_RANGE = 0x2
DEVERR_NONFINITE = 0x4
DEVERR_SEQLEN_RANGE = 0x8
DEVERR_TIMEOUT = 0x10
DEVERR_LAYOUT = 0x20

EXPORTED = ("tq_slot_bytes", "tq_quantize_append", "tq_paged_decode", "tq_paged_decode_hot",
            "tq_paged_decode_noalloc",
            "tq_decode_workspace_size", "tq_set_workspace", "tq_get_device_error",
            "tq_rotate_unit", "tq_decode_plan_probe", "tq_debug_inject_merge_stall",
            "tq_quantize_append_dense", "tq_paged_decode_dense", "tq_rotate_unit_dense",
            "tq_slot_bytes_qjl", "tq_quantize_append_qjl", "tq_paged_decode_qjl",
            "tq_status_string", "tq_version")


class TQError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


class TensorDesc(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class CodebookDesc(ctypes.Structure):
    _fields_ = [("dim", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("centroids", ctypes.c_void_p), ("boundaries", ctypes.c_void_p)]


class CodebooksDesc(ctypes.Structure):
    _fields_ = [("k", CodebookDesc), ("v", CodebookDesc)]


class RotationDesc(ctypes.Structure):
    _fields_ = [("dim", ctypes.c_int32), ("hi", ctypes.c_void_p), ("lo", ctypes.c_void_p)]


_lib = None


def library_path() -> str:
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing: build it with `python -m kv_cache_vector_append_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(_LIB_PATH)
    T, CB = TensorDesc, ctypes.POINTER(CodebooksDesc)
    RT = ctypes.POINTER(RotationDesc)
    sig = {
        "tq_slot_bytes": [ctypes.c_int32] * 3 + [ctypes.POINTER(ctypes.c_int32)],
        "tq_quantize_append": [T, T, T, T, CB, ctypes.c_uint64, ctypes.c_int32, ctypes.c_int32,
                               ctypes.c_void_p],
        "tq_paged_decode": [T, T, T, T, T, CB, ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p],
        "tq_paged_decode_noalloc": [T, T, T, T, T, CB, ctypes.c_uint64, ctypes.c_float,
                                    ctypes.c_void_p],
        "tq_paged_decode_hot": [T, T, T, T, T, T, T, T, CB, ctypes.c_uint64, ctypes.c_float,
                                ctypes.c_void_p],
        "tq_decode_workspace_size": [ctypes.c_int32] * 6 + [ctypes.POINTER(ctypes.c_size_t)],
        "tq_set_workspace": [ctypes.c_void_p, ctypes.c_size_t],
        "tq_get_device_error": [ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p],
        "tq_rotate_unit": [T, T, T, ctypes.c_uint64, ctypes.c_void_p],
        "tq_decode_plan_probe": [ctypes.c_int32] * 10 + [ctypes.c_uint32,
                                                         ctypes.POINTER(ctypes.c_int64)],
        "tq_debug_inject_merge_stall": [ctypes.c_int32, ctypes.c_int32],
        "tq_quantize_append_dense": [T, T, T, T, CB, RT, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_void_p],
        "tq_paged_decode_dense": [T, T, T, T, T, CB, RT, ctypes.c_float, ctypes.c_void_p],
        "tq_rotate_unit_dense": [T, T, T, RT, ctypes.c_void_p],
        "tq_slot_bytes_qjl": [ctypes.c_int32] * 3 + [ctypes.POINTER(ctypes.c_int32)],
        "tq_quantize_append_qjl": [T, T, T, T, CB, ctypes.c_uint64, ctypes.c_uint64,
                                   ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p],
        "tq_paged_decode_qjl": [T, T, T, T, T, CB, ctypes.c_uint64, ctypes.c_uint64,
                                ctypes.c_float, ctypes.c_void_p],
        "tq_status_string": [ctypes.c_int],
    }
    for name, args in sig.items():
        fn = getattr(lib, name, None)     # every declared symbol is checked by the ABI test
        if fn is None:
            continue
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name == "tq_status_string" else ctypes.c_int
    lib.tq_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return _load().tq_status_string(int(status)).decode()


def version() -> str:
    return _load().tq_version().decode()


def _check(status: int, what: str) -> None:
    if status != OK:
        raise TQError(status, what)


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    table = {torch.uint8: U8, torch.int32: I32, torch.int64: I64, torch.float32: F32,
             torch.bfloat16: BF16, torch.float16: F16}
    if t.dtype not in table:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return table[t.dtype]


def _desc(t) -> TensorDesc:
    if t.dim() > 4:
        raise ValueError("tensors of rank > 4 are not supported")
    d = TensorDesc()
    d.data = t.data_ptr()
    d.dtype = _dtype_code(t)
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def _stream_handle(stream, device):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _require_cuda(*tensors):
    for t in tensors:
        if not t.is_cuda:
            raise ValueError("all tensors must live on a CUDA device (no CPU fallback)")


# ---------------------------------------------------------------------------
# Codebooks
# ---------------------------------------------------------------------------

@dataclass
class CodebookTable:
    """One fp32 Lloyd-Max table read from the library's data files."""
    dim: int
    bits: int
    centroids: np.ndarray
    boundaries: np.ndarray


CODEBOOK_KINDS = ("beta", "gauss")


def load_codebook_table(dim: int, bits: int, kind: str = "beta") -> CodebookTable:
    """Read ``codebooks/{kind}_d{dim}_b{bits}.tqcb`` (magic, 7 u32, L f32, L-1 f32):
    kind "beta" is the exact Beta-sphere table, "gauss" its Gaussian approximation
    N(0, 1/D) (TorbuQuant, "Current Status")."""
    if kind not in CODEBOOK_KINDS:
        raise ValueError(f"codebook kind {kind!r}: one of {CODEBOOK_KINDS}")
    path = os.path.join(_CODEBOOK_DIR, f"{kind}_d{dim}_b{bits}.tqcb")
    with open(path, "rb") as f:
        raw = f.read()
    if raw[:4] != b"TQCB":
        raise ValueError(f"{path}: not a codebook table")
    version_, d, b, _dens, _n_iter, _iters, _ = struct.unpack_from("<7I", raw, 4)
    if version_ != 1 or d != dim or b != bits:
        raise ValueError(f"{path}: unexpected header")
    levels = 1 << bits
    c = np.frombuffer(raw, dtype="<f4", count=levels, offset=32).copy()
    bnd = np.frombuffer(raw, dtype="<f4", count=levels - 1, offset=32 + 4 * levels).copy()
    return CodebookTable(dim, bits, c, bnd)


class Codebooks:
    """Device-resident K and V tables plus the C descriptor that points at them."""

    def __init__(self, dim: int, k_bits: int, v_bits: int, device="cuda", kind: str = "beta"):
        torch = _torch()
        self.dim, self.k_bits, self.v_bits, self.kind = dim, k_bits, v_bits, kind
        self.k_table = load_codebook_table(dim, k_bits, kind)
        self.v_table = load_codebook_table(dim, v_bits, kind)
        self.k_centroids = torch.from_numpy(self.k_table.centroids).to(device)
        self.k_boundaries = torch.from_numpy(self.k_table.boundaries).to(device)
        if v_bits == k_bits:
            self.v_centroids, self.v_boundaries = self.k_centroids, self.k_boundaries
        else:
            self.v_centroids = torch.from_numpy(self.v_table.centroids).to(device)
            self.v_boundaries = torch.from_numpy(self.v_table.boundaries).to(device)
        self.desc = CodebooksDesc()
        self.desc.k = CodebookDesc(dim, k_bits, self.k_centroids.data_ptr(),
                                   self.k_boundaries.data_ptr())
        self.desc.v = CodebookDesc(dim, v_bits, self.v_centroids.data_ptr(),
                                   self.v_boundaries.data_ptr())


_ROTATION_DIR = os.path.join(_PKG, "rotations")


class Rotation:
    """Device copy of the dense rotation table ``rotations/qr_d{dim}.tqrt`` (magic, 3 u32,
    then hi and lo as D*D bf16 bit patterns each) and the C descriptor pointing at it."""

    def __init__(self, dim: int, device="cuda"):
        torch = _torch()
        path = os.path.join(_ROTATION_DIR, f"qr_d{dim}.tqrt")
        with open(path, "rb") as f:
            raw = f.read()
        if raw[:4] != b"TQRT":
            raise ValueError(f"{path}: not a rotation table")
        version_, d, self.seed = struct.unpack_from("<3I", raw, 4)
        if version_ != 1 or d != dim:
            raise ValueError(f"{path}: unexpected header")
        words = np.frombuffer(raw, dtype="<u2", count=2 * dim * dim, offset=16).copy()
        self.dim = dim
        w = torch.from_numpy(words.view(np.int16)).to(device)
        self.hi = w[:dim * dim].contiguous()
        self.lo = w[dim * dim:].contiguous()
        self.desc = RotationDesc(dim, self.hi.data_ptr(), self.lo.data_ptr())


def load_rotation(dim: int, device="cuda") -> Rotation:
    return Rotation(dim, device)


def load_codebooks(dim: int, k_bits: int, v_bits: int, device="cuda",
                   kind: str = "beta") -> Codebooks:
    return Codebooks(dim, k_bits, v_bits, device, kind)


# ---------------------------------------------------------------------------
# Entry points
# ---------------------------------------------------------------------------

def slot_bytes(dim: int, k_bits: int, v_bits: int) -> int:
    out = ctypes.c_int32()
    _check(_load().tq_slot_bytes(dim, k_bits, v_bits, ctypes.byref(out)), "tq_slot_bytes")
    return out.value


def quantize_append(pages, slot_mapping, k, v, codebooks: Codebooks, sign_seed: int,
                    stream=None) -> None:
    _require_cuda(pages, slot_mapping, k, v)
    st = _stream_handle(stream, pages.device)
    _check(_load().tq_quantize_append(_desc(pages), _desc(slot_mapping), _desc(k), _desc(v),
                                      ctypes.byref(codebooks.desc), ctypes.c_uint64(sign_seed),
                                      codebooks.k_bits, codebooks.v_bits, st),
           "tq_quantize_append")


def paged_decode(out, q, pages, block_table, seq_lens, codebooks: Codebooks, sign_seed: int,
                 scale: float, stream=None) -> None:
    _require_cuda(out, q, pages, block_table, seq_lens)
    st = _stream_handle(stream, q.device)
    _check(_load().tq_paged_decode(_desc(out), _desc(q), _desc(pages), _desc(block_table),
                                   _desc(seq_lens), ctypes.byref(codebooks.desc),
                                   ctypes.c_uint64(sign_seed), ctypes.c_float(scale), st),
           "tq_paged_decode")


def paged_decode_hot(out, q, pages, block_table, seq_lens, hot_k, hot_v, hot_lens,
                     codebooks: Codebooks, sign_seed: int, scale: float, stream=None) -> None:
    """tq_paged_decode_hot: the decode over the packed pages plus an uncompressed hot
    window hot_k/hot_v [B, W, H_kv, D] holding hot_lens[b] tokens of sequence b."""
    _require_cuda(out, q, pages, block_table, seq_lens, hot_k, hot_v, hot_lens)
    st = _stream_handle(stream, q.device)
    _check(_load().tq_paged_decode_hot(_desc(out), _desc(q), _desc(pages), _desc(block_table),
                                       _desc(seq_lens), _desc(hot_k), _desc(hot_v),
                                       _desc(hot_lens), ctypes.byref(codebooks.desc),
                                       ctypes.c_uint64(sign_seed), ctypes.c_float(scale), st),
           "tq_paged_decode_hot")


NOALLOC_SCRATCH_BYTES = 16 << 20


def paged_decode_noalloc(out, q, pages, block_table, seq_lens, codebooks: Codebooks,
                         sign_seed: int, scale: float, stream=None) -> None:
    """tq_paged_decode_noalloc: the decode with the library's fixed scratch array
    (no device allocation on the call path; see include/tq.h)."""
    _require_cuda(out, q, pages, block_table, seq_lens)
    st = _stream_handle(stream, q.device)
    _check(_load().tq_paged_decode_noalloc(_desc(out), _desc(q), _desc(pages), _desc(block_table),
                                           _desc(seq_lens), ctypes.byref(codebooks.desc),
                                           ctypes.c_uint64(sign_seed), ctypes.c_float(scale), st),
           "tq_paged_decode_noalloc")


def quantize_append_dense(pages, slot_mapping, k, v, codebooks: Codebooks, rotation: Rotation,
                          stream=None) -> None:
    _require_cuda(pages, slot_mapping, k, v)
    st = _stream_handle(stream, pages.device)
    _check(_load().tq_quantize_append_dense(_desc(pages), _desc(slot_mapping), _desc(k),
                                            _desc(v), ctypes.byref(codebooks.desc),
                                            ctypes.byref(rotation.desc), codebooks.k_bits,
                                            codebooks.v_bits, st),
           "tq_quantize_append_dense")


def paged_decode_dense(out, q, pages, block_table, seq_lens, codebooks: Codebooks,
                       rotation: Rotation, scale: float, stream=None) -> None:
    _require_cuda(out, q, pages, block_table, seq_lens)
    st = _stream_handle(stream, q.device)
    _check(_load().tq_paged_decode_dense(_desc(out), _desc(q), _desc(pages), _desc(block_table),
                                         _desc(seq_lens), ctypes.byref(codebooks.desc),
                                         ctypes.byref(rotation.desc), ctypes.c_float(scale), st),
           "tq_paged_decode_dense")


def rotate_unit_dense(u, norm, x, rotation: Rotation, stream=None) -> None:
    _require_cuda(u, norm, x)
    st = _stream_handle(stream, x.device)
    _check(_load().tq_rotate_unit_dense(_desc(u), _desc(norm), _desc(x),
                                        ctypes.byref(rotation.desc), st),
           "tq_rotate_unit_dense")


def slot_bytes_qjl(dim: int, k_bits: int, v_bits: int) -> int:
    out = ctypes.c_int32()
    _check(_load().tq_slot_bytes_qjl(dim, k_bits, v_bits, ctypes.byref(out)), "tq_slot_bytes_qjl")
    return out.value


def quantize_append_qjl(pages, slot_mapping, k, v, codebooks: Codebooks, sign_seed: int,
                        qjl_seed: int, stream=None) -> None:
    _require_cuda(pages, slot_mapping, k, v)
    st = _stream_handle(stream, pages.device)
    _check(_load().tq_quantize_append_qjl(_desc(pages), _desc(slot_mapping), _desc(k), _desc(v),
                                          ctypes.byref(codebooks.desc), ctypes.c_uint64(sign_seed),
                                          ctypes.c_uint64(qjl_seed), codebooks.k_bits,
                                          codebooks.v_bits, st),
           "tq_quantize_append_qjl")


def paged_decode_qjl(out, q, pages, block_table, seq_lens, codebooks: Codebooks, sign_seed: int,
                     qjl_seed: int, scale: float, stream=None) -> None:
    _require_cuda(out, q, pages, block_table, seq_lens)
    st = _stream_handle(stream, q.device)
    _check(_load().tq_paged_decode_qjl(_desc(out), _desc(q), _desc(pages), _desc(block_table),
                                       _desc(seq_lens), ctypes.byref(codebooks.desc),
                                       ctypes.c_uint64(sign_seed), ctypes.c_uint64(qjl_seed),
                                       ctypes.c_float(scale), st),
           "tq_paged_decode_qjl")


def rotate_unit(u, norm, x, sign_seed: int, stream=None) -> None:
    _require_cuda(u, norm, x)
    st = _stream_handle(stream, x.device)
    _check(_load().tq_rotate_unit(_desc(u), _desc(norm), _desc(x), ctypes.c_uint64(sign_seed), st),
           "tq_rotate_unit")


DECODE_PLAN_FIELDS = ("wph", "nst", "row_pitch", "stage_bytes", "lut_win", "lut_off", "lut_bytes",
                      "stage_lo_off", "stage_hi_off", "n_low", "misc_off", "smem", "copy_mode",
                      "warps")


def decode_plan_probe(batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                      k_bits: int, v_bits: int, slot_stride: int, max_blocks: int,
                      num_sms: int, max_smem_optin: int, dyn_smem_base: int):
    """Host-only test export: the decode kernel's shared-memory plan as a dict, or the
    status code when no plan is returned."""
    out = (ctypes.c_int64 * len(DECODE_PLAN_FIELDS))()
    s = _load().tq_decode_plan_probe(batch, num_q_heads, num_kv_heads, head_dim, k_bits, v_bits,
                                     slot_stride, max_blocks, num_sms, max_smem_optin,
                                     dyn_smem_base, out)
    return dict(zip(DECODE_PLAN_FIELDS, list(out))) if s == OK else s


def debug_inject_merge_stall(withhold_cta: int, wait_ms: int) -> None:
    """Test export: the next decode launch on the current device waits at most
    ``wait_ms`` ms and its CTA ``withhold_cta`` never announces its partial results
    (see include/tq.h)."""
    _check(_load().tq_debug_inject_merge_stall(withhold_cta, wait_ms),
           "tq_debug_inject_merge_stall")


def decode_workspace_size(batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                          max_blocks: int, block_size: int = 16) -> int:
    out = ctypes.c_size_t()
    _check(_load().tq_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim,
                                            max_blocks, block_size, ctypes.byref(out)),
           "tq_decode_workspace_size")
    return out.value


def set_workspace(tensor) -> None:
    """Hand a caller-owned device buffer (any dtype, contiguous) to the library
    for the current device, or ``None`` to release it."""
    if tensor is None:
        _check(_load().tq_set_workspace(None, 0), "tq_set_workspace")
        return
    _require_cuda(tensor)
    _check(_load().tq_set_workspace(ctypes.c_void_p(tensor.data_ptr()),
                                    tensor.numel() * tensor.element_size()), "tq_set_workspace")


def get_device_error(stream=None) -> int:
    torch = _torch()
    out = ctypes.c_int32()
    st = _stream_handle(stream, torch.cuda.current_device())
    _check(_load().tq_get_device_error(ctypes.byref(out), st), "tq_get_device_error")
    return out.value
