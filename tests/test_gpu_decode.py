"""GPU parity of tq_paged_decode against the oracle's dequantize-then-attend
over the same (GPU-written) pages."""
import numpy as np
import pytest
import torch

from oracle import tq_oracle as O
from kv_cache_vector_append_b200 import workloads as W
from tests.gpu_helpers import (decode_error, gpu_append, gpu_decode, oracle_table, require_gpu,
                               to_np_f64)

pytestmark = pytest.mark.gpu
TOL = 2e-3   # max_{b,h} ||o_gpu - o_ref||_inf / ||o_ref||_2


def _tq():
    require_gpu()
    import kv_cache_vector_append_b200 as tq
    return tq


def _oracle_decode(wl, pages_np, seqs=None):
    d = wl.spec.head_dim
    kt, vt = oracle_table(d, wl.spec.k_bits), oracle_table(d, wl.spec.v_bits)
    seqs = np.arange(wl.spec.batch) if seqs is None else np.asarray(seqs)
    q = to_np_f64(wl.q)[seqs]
    return O.paged_decode(q, pages_np, wl.block_table[seqs], wl.seq_lens[seqs], kt, vt,
                          wl.spec.sign_seed, wl.spec.scale)


def _case(tq, wl, out_dtype=None, seqs=None):
    pages, cb = gpu_append(tq, wl)
    out = gpu_decode(tq, wl, pages, cb, out_dtype)
    ref = _oracle_decode(wl, pages.cpu().numpy(), seqs)
    got = to_np_f64(out)
    if seqs is not None:
        got = got[np.asarray(seqs)]
    err = decode_error(got, ref)
    assert err <= TOL, err
    return err


def _spec(d, h_q, h_kv, kb, vb, lens, dtype="bfloat16", seed=11):
    lens = list(lens)
    return W.WorkloadSpec(f"mini-d{d}-g{h_q // h_kv}", d, h_q, h_kv, len(lens), kb, vb, dtype,
                          seq_len=max(lens), n_outliers=2, outlier_factor=20.0, seed=seed)


def _with_lens(spec, lens):
    # regenerate with ragged lengths: same recipe, then override the lengths by
    # building a workload per the maximum and masking through seq_lens.
    wl = W.generate(spec)
    wl.seq_lens = np.asarray(lens, dtype=np.int32)
    return wl


def test_config0():
    tq = _tq()
    _case(tq, W.generate(W.CONFIGS[0]))


@pytest.mark.parametrize("d,h_q,h_kv,kb,vb", [
    (128, 32, 8, 4, 4), (64, 14, 2, 8, 8), (128, 28, 4, 4, 2), (128, 32, 8, 3, 2),
    (128, 8, 8, 4, 4), (256, 8, 2, 4, 4), (64, 4, 1, 2, 2), (128, 12, 1, 3, 3),
    (128, 16, 1, 8, 4), (256, 16, 4, 4, 3), (64, 6, 2, 4, 4)])
def test_mini_geometries(d, h_q, h_kv, kb, vb):
    tq = _tq()
    lens = [300, 17, 64]
    _case(tq, _with_lens(_spec(d, h_q, h_kv, kb, vb, lens), lens))


def test_ragged_and_edge_lengths():
    tq = _tq()
    spec = _spec(128, 8, 2, 4, 2, [129] * 8)
    wl = _with_lens(spec, [0, 1, 15, 16, 17, 33, 128, 129])
    pages, cb = gpu_append(tq, wl)
    out = gpu_decode(tq, wl, pages, cb)
    ref = _oracle_decode(wl, pages.cpu().numpy())
    got = to_np_f64(out)
    assert np.all(got[0] == 0.0)                       # empty sequence
    assert decode_error(got, ref) <= TOL


def test_fp32_output_and_long_split():
    tq = _tq()
    wl = W.generate(_spec(128, 8, 2, 4, 4, [5000, 2000], seed=3))
    _case(tq, wl, out_dtype=torch.float32)


def test_block_table_out_of_range_flagged():
    tq = _tq()
    wl = W.generate(_spec(128, 4, 1, 4, 4, [64, 64]))
    pages, cb = gpu_append(tq, wl)
    wl.block_table[1, 2] = wl.num_blocks + 3
    tq.get_device_error()
    gpu_decode(tq, wl, pages, cb)
    assert tq.get_device_error() & tq.DEVERR_BLOCK_RANGE
    wl.seq_lens[0] = 10_000
    gpu_decode(tq, wl, pages, cb)
    assert tq.get_device_error() & tq.DEVERR_SEQLEN_RANGE


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_full_size_configs_sampled(cfg):
    # Full-size append and decode in the bench's launch configuration; the oracle
    # recomputes a seeded sample of sequences.
    tq = _tq()
    wl = W.generate(W.CONFIGS[cfg])
    pages, cb = gpu_append(tq, wl)
    out = gpu_decode(tq, wl, pages, cb)
    rng = np.random.default_rng(cfg)
    seqs = np.sort(rng.choice(wl.spec.batch, size=min(2, wl.spec.batch), replace=False))
    ref = _oracle_decode(wl, pages.cpu().numpy(), seqs)
    err = decode_error(to_np_f64(out)[seqs], ref)
    assert err <= TOL, err
