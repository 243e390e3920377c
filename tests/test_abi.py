"""CPU checks of the C-ABI library: it loads, exports every symbol the header
declares, and its host-side logic (slot formula, argument validation) works
without a GPU."""
import ctypes
import os
import re

import pytest
import torch

from oracle import tq_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib():
    import kv_cache_vector_append_b200 as tq
    from kv_cache_vector_append_b200 import _binding as B
    return tq, B, B._load()


def test_library_exports_every_declared_symbol():
    tq, B, lib = _lib()
    header = open(os.path.join(ROOT, "include", "tq.h")).read()
    declared = re.findall(r"TQ_API\s+[\w\s\*]+?\b(tq_\w+)\s*\(", header)
    assert len(declared) >= 9
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(B.EXPORTED)
    assert tq.version() == "0.1.0"


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kb,vb", [(4, 4), (8, 8), (4, 2), (3, 2), (1, 8), (5, 7)])
def test_slot_bytes_matches_oracle(d, kb, vb):
    tq, _, _ = _lib()
    assert tq.slot_bytes(d, kb, vb) == O.slot_bytes(d, kb, vb)


def test_status_strings_and_bad_slot_args():
    tq, B, lib = _lib()
    for s in range(7):
        assert isinstance(B.status_string(s), str)
    out = ctypes.c_int32()
    assert lib.tq_slot_bytes(128, 0, 4, ctypes.byref(out)) == B.ERR_INVALID_ARG
    assert lib.tq_slot_bytes(128, 4, 9, ctypes.byref(out)) == B.ERR_INVALID_ARG
    assert lib.tq_slot_bytes(128, 4, 4, None) == B.ERR_INVALID_ARG


def _fake(shape, dtype, strides=None, ptr=0x10000):
    d = __import__("kv_cache_vector_append_b200._binding", fromlist=["x"]).TensorDesc()
    d.data = ptr
    d.dtype = dtype
    d.ndim = len(shape)
    st = strides or [int(x) for x in torch.empty(shape).stride()] if len(shape) else []
    for i, n in enumerate(shape):
        d.shape[i] = n
        d.stride[i] = st[i]
    return d


def test_host_validation_rejects_before_touching_the_device():
    # Every case below fails host validation, so no CUDA call is made (this runs
    # on a machine without a GPU).
    tq, B, lib = _lib()
    cbs = B.CodebooksDesc()
    cbs.k = B.CodebookDesc(128, 4, 0x20000, 0x30000)
    cbs.v = B.CodebookDesc(128, 4, 0x40000, 0x50000)
    pages = _fake([4, 16, 2, 136], B.U8)
    sm = _fake([10], B.I64)
    k = _fake([10, 2, 128], B.BF16)
    v = _fake([10, 2, 128], B.BF16)
    ok_args = dict(pages=pages, sm=sm, k=k, v=v)

    def app(pages=pages, sm=sm, k=k, v=v, cb=cbs, kb=4, vb=4):
        return lib.tq_quantize_append(pages, sm, k, v, ctypes.byref(cb) if cb is not None else None,
                                      0, kb, vb, None)

    assert app(cb=None) == B.ERR_INVALID_ARG
    assert app(kb=3) == B.ERR_INVALID_ARG                       # bits != codebook bits
    assert app(pages=_fake([4, 16, 2, 100], B.U8)) == B.ERR_INVALID_ARG   # slot too small
    assert app(pages=_fake([4, 16, 3, 136], B.U8)) == B.ERR_INVALID_ARG   # H_kv mismatch
    assert app(sm=_fake([9], B.I64)) == B.ERR_INVALID_ARG
    assert app(sm=_fake([10], B.I32)) == B.ERR_INVALID_ARG
    assert app(v=_fake([10, 2, 128], B.F32)) == B.ERR_INVALID_ARG       # dtype mismatch
    bad = B.CodebooksDesc()
    bad.k = B.CodebookDesc(64, 4, 0x20000, 0x30000)
    bad.v = cbs.v
    assert app(cb=bad) == B.ERR_INVALID_ARG                     # codebook dim != D
    k96 = _fake([10, 2, 96], B.BF16)
    cb96 = B.CodebooksDesc()
    cb96.k = B.CodebookDesc(96, 4, 0x20000, 0x30000)
    cb96.v = B.CodebookDesc(96, 4, 0x20000, 0x30000)
    assert app(k=k96, v=k96, cb=cb96, pages=_fake([4, 16, 2, 104], B.U8)) == B.ERR_UNSUPPORTED

    q = _fake([2, 8, 128], B.BF16)
    out = _fake([2, 8, 128], B.BF16)
    bt = _fake([2, 4], B.I32)
    sl = _fake([2], B.I32)

    def dec(out=out, q=q, pages=pages, bt=bt, sl=sl, cb=cbs, scale=0.1):
        return lib.tq_paged_decode(out, q, pages, bt, sl, ctypes.byref(cb), 0, scale, None)

    assert dec(scale=float("nan")) == B.ERR_INVALID_ARG
    assert dec(out=_fake([2, 8, 128], B.F16)) == B.ERR_INVALID_ARG      # out dtype
    assert dec(q=_fake([2, 7, 128], B.BF16), out=_fake([2, 7, 128], B.BF16)) == B.ERR_INVALID_ARG
    assert dec(bt=_fake([3, 4], B.I32)) == B.ERR_INVALID_ARG
    assert dec(sl=_fake([2], B.I64)) == B.ERR_INVALID_ARG
    assert dec(pages=_fake([4, 8, 2, 136], B.U8)) == B.ERR_UNSUPPORTED   # block size 8
    assert dec(pages=_fake([4, 16, 2, 136], B.U8, strides=[4352 * 2, 272, 136, 1])) == \
        B.ERR_INVALID_ARG                                               # non-contiguous
    big_g = _fake([2, 34, 128], B.BF16)
    assert dec(q=big_g, out=big_g) == B.ERR_UNSUPPORTED                 # G = 17 > 16
    odd = B.CodebooksDesc()
    odd.k = B.CodebookDesc(128, 5, 0x20000, 0x30000)
    odd.v = B.CodebookDesc(128, 7, 0x20000, 0x30000)
    assert dec(cb=odd, pages=_fake([4, 16, 2, 200], B.U8)) == B.ERR_UNSUPPORTED


def test_binding_refuses_cpu_tensors():
    tq, _, _ = _lib()
    cpu = torch.zeros(4, 16, 1, 136, dtype=torch.uint8)
    with pytest.raises(ValueError):
        tq.quantize_append(cpu, torch.zeros(1, dtype=torch.int64), torch.zeros(1, 1, 128),
                           torch.zeros(1, 1, 128), None, 0)


def test_host_limits_and_empty_inputs_on_cpu():
    # Limits and empty inputs are settled by host validation alone (no GPU here).
    tq, B, lib = _lib()
    cbs = B.CodebooksDesc()
    cbs.k = B.CodebookDesc(128, 4, 0x20000, 0x30000)
    cbs.v = B.CodebookDesc(128, 4, 0x40000, 0x50000)

    def app(pages, sm, k, v):
        return lib.tq_quantize_append(pages, sm, k, v, ctypes.byref(cbs), 0, 4, 4, None)

    # no tokens: nothing to do, success without touching the device
    empty = _fake([0, 2, 128], B.BF16, strides=[256, 128, 1])
    assert app(_fake([4, 16, 2, 136], B.U8), _fake([0], B.I64, strides=[1]), empty, empty) == B.OK
    # 2^28 tokens x 8 heads reaches the 32-bit row-index limit
    t = 1 << 28
    big = _fake([t, 8, 128], B.BF16, strides=[1024, 128, 1])
    assert app(_fake([4, 16, 8, 136], B.U8, strides=[17408, 1088, 136, 1]),
               _fake([t], B.I64, strides=[1]), big, big) == B.ERR_UNSUPPORTED
    # slot stride must be a multiple of 8 bytes
    k = _fake([10, 2, 128], B.BF16)
    assert app(_fake([4, 16, 2, 140], B.U8), _fake([10], B.I64), k, k) == B.ERR_INVALID_ARG

    def dec(h_q, h_kv, d, cb):
        q = _fake([2, h_q, d], B.BF16, strides=[h_q * d, d, 1])
        pages = _fake([4, 16, h_kv, 136 if d == 128 else 264], B.U8,
                      strides=[16 * h_kv * (136 if d == 128 else 264), h_kv * (136 if d == 128 else 264),
                               136 if d == 128 else 264, 1])
        return lib.tq_paged_decode(q, q, pages, _fake([2, 4], B.I32), _fake([2], B.I32),
                                   ctypes.byref(cb), 0, 0.1, None)

    # more KV heads than the decode kernel's warps: 32 at D=128, 16 at D=256
    assert dec(32, 32, 128, cbs) == B.ERR_UNSUPPORTED
    cb256 = B.CodebooksDesc()
    cb256.k = B.CodebookDesc(256, 4, 0x20000, 0x30000)
    cb256.v = B.CodebookDesc(256, 4, 0x40000, 0x50000)
    assert dec(16, 16, 256, cb256) == B.ERR_UNSUPPORTED
