"""Failure detection of the decode without a GPU fault.

A test hook makes one CTA of the next decode launch withhold the announcement of
its partial results (a flag that nothing else sets) and shortens every bounded wait
to 20 ms.  The CTAs that share its sequence must give up waiting, report
TQ_DEVERR_TIMEOUT through the error word, and leave the merge counters at zero: the
next, normal call is checked BEFORE the error word is read (reading it would clear the
counters on the host side), so it proves the kernel's own clean-up.
"""
import numpy as np
import pytest
import torch

from kv_cache_vector_append_b200 import workloads as W
from tests.gpu_helpers import decode_error, gpu_append, require_gpu, to_np_f64
from tests.test_gpu_decode import TOL, _oracle_decode

pytestmark = pytest.mark.gpu


def _tq():
    require_gpu()
    import kv_cache_vector_append_b200 as tq
    return tq


def _workload():
    # one long sequence spans many CTAs (CTA 0 covers its first steps), plus a short one
    spec = W.WorkloadSpec("stall", 128, 8, 2, 2, 4, 4, "bfloat16", seq_len=6000,
                          n_outliers=2, outlier_factor=20.0, seed=31)
    wl = W.generate(spec)
    wl.seq_lens = np.array([6000, 300], dtype=np.int32)
    return wl


@pytest.mark.parametrize("entry", ["paged_decode", "paged_decode_noalloc"])
def test_withheld_arrival_times_out_and_the_next_call_is_clean(entry):
    tq = _tq()
    wl = _workload()
    pages, cb = gpu_append(tq, wl)
    q = wl.q.cuda()
    bt = torch.from_numpy(wl.block_table).cuda()
    sl = torch.from_numpy(wl.seq_lens).cuda()
    call = getattr(tq, entry)
    assert tq.get_device_error() == 0
    stalled = torch.zeros(q.shape, dtype=torch.float32, device="cuda")
    tq.debug_inject_merge_stall(0, 20)
    call(stalled, q, pages, bt, sl, cb, wl.spec.sign_seed, wl.spec.scale)
    # the next call runs on the counters the stalled launch left behind
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    call(out, q, pages, bt, sl, cb, wl.spec.sign_seed, wl.spec.scale)
    torch.cuda.synchronize()
    err = tq.get_device_error()
    assert err & tq.DEVERR_TIMEOUT, hex(err)
    ref = _oracle_decode(wl, pages.cpu().numpy())
    got = to_np_f64(out)
    assert np.all(np.isfinite(got))
    assert decode_error(got, ref) <= TOL
    # and once more after the error word was read
    out.fill_(float("nan"))
    call(out, q, pages, bt, sl, cb, wl.spec.sign_seed, wl.spec.scale)
    torch.cuda.synchronize()
    assert tq.get_device_error() == 0
    assert decode_error(to_np_f64(out), ref) <= TOL


def test_hook_rejects_bad_arguments():
    tq = _tq()
    from kv_cache_vector_append_b200 import _binding as B
    for args in ((-1, 20), (0, 0), (0, 5000)):
        with pytest.raises(B.TQError):
            tq.debug_inject_merge_stall(*args)
