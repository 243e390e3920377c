"""GPU test of tq_paged_decode_noalloc, the decode entry point that allocates no
device memory (it uses the library's fixed scratch array).

Some callers cannot let a library allocate on the call path: a serving loop that
keeps cudaMalloc/cudaFree (which can synchronise the device) out of its steady
state, or a runtime that owns all device memory itself.  This checks that the
allocation-free entry point gives the same results as tq_paged_decode, on
consecutive calls that share (and leave stale data in) the one scratch array, and
that it refuses a geometry whose scratch would not fit.  Named so that pytest runs
it after every other test file.
"""
import numpy as np
import pytest
import torch

from kv_cache_vector_append_b200 import workloads as W
from tests.gpu_helpers import decode_error, gpu_append, require_gpu, to_np_f64

pytestmark = pytest.mark.gpu
TOL = 2e-3   # same bound as the decode parity tests


def _tq():
    require_gpu()
    import kv_cache_vector_append_b200 as tq
    return tq


def _workload(d, h_q, h_kv, kb, vb, lens, seed):
    spec = W.WorkloadSpec("noalloc", d, h_q, h_kv, len(lens), kb, vb, "bfloat16",
                          seq_len=max(lens), n_outliers=2, outlier_factor=20.0, seed=seed)
    wl = W.generate(spec)
    wl.seq_lens = np.asarray(lens, dtype=np.int32)
    return wl


def _both(tq, wl):
    pages, cb = gpu_append(tq, wl)
    q = wl.q.cuda()
    bt = torch.from_numpy(wl.block_table).cuda()
    sl = torch.from_numpy(wl.seq_lens).cuda()
    ref = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    tq.paged_decode(ref, q, pages, bt, sl, cb, wl.spec.sign_seed, wl.spec.scale)
    got = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    tq.paged_decode_noalloc(got, q, pages, bt, sl, cb, wl.spec.sign_seed, wl.spec.scale)
    torch.cuda.synchronize()
    return to_np_f64(got), to_np_f64(ref)


def test_noalloc_matches_decode_on_consecutive_calls():
    tq = _tq()
    a = _workload(128, 8, 2, 4, 2, [300, 17, 64, 1, 0], seed=21)
    b = _workload(64, 14, 2, 8, 8, [129, 1000, 33], seed=22)
    for wl in (a, b, a):          # the scratch keeps the previous call's contents
        got, ref = _both(tq, wl)
        assert np.all(np.isfinite(got))
        assert decode_error(got, ref) <= TOL
    assert tq.get_device_error() == 0


def test_noalloc_rejects_oversized_geometry():
    tq = _tq()
    from kv_cache_vector_append_b200 import _binding as B
    # 4096 sequences x 32 query heads of partial records exceed the fixed scratch
    bsz, h_q, h_kv, d = 4096, 32, 8, 128
    need = tq.decode_workspace_size(bsz, h_q, h_kv, d, 1)
    assert need > B.NOALLOC_SCRATCH_BYTES
    cb = tq.load_codebooks(d, 4, 4, "cuda")
    pages = torch.zeros(2, 16, h_kv, tq.slot_bytes(d, 4, 4), dtype=torch.uint8, device="cuda")
    q = torch.zeros(bsz, h_q, d, dtype=torch.bfloat16, device="cuda")
    out = torch.full((bsz, h_q, d), 7.0, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(bsz, 1, dtype=torch.int32, device="cuda")
    sl = torch.ones(bsz, dtype=torch.int32, device="cuda")
    with pytest.raises(B.TQError) as e:
        tq.paged_decode_noalloc(out, q, pages, bt, sl, cb, 0, 0.1)
    assert e.value.status == B.ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)     # nothing was enqueued
