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


def _oracle_decode(wl, pages_np, seqs=None, kind="beta"):
    d = wl.spec.head_dim
    kt, vt = oracle_table(d, wl.spec.k_bits, kind), oracle_table(d, wl.spec.v_bits, kind)
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
    # recomputes a seeded sample of 8 sequences that always holds the shortest and the
    # longest one (all of them when the batch is smaller).
    tq = _tq()
    wl = W.generate(W.CONFIGS[cfg])
    pages, cb = gpu_append(tq, wl)
    out = gpu_decode(tq, wl, pages, cb)
    rng = np.random.default_rng(cfg)
    bsz = wl.spec.batch
    pick = {int(np.argmin(wl.seq_lens)), int(np.argmax(wl.seq_lens))}
    rest = [b for b in rng.permutation(bsz) if b not in pick]
    seqs = np.sort(np.array(sorted(pick) + rest[:max(0, min(8, bsz) - len(pick))]))
    ref = _oracle_decode(wl, pages.cpu().numpy(), seqs)
    err = decode_error(to_np_f64(out)[seqs], ref)
    assert err <= TOL, err


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kb", [2, 3, 4, 8])
@pytest.mark.parametrize("vb", [2, 3, 4, 8])
def test_every_required_bit_pair(d, kb, vb):
    tq = _tq()
    lens = [200, 17, 33]
    _case(tq, _with_lens(_spec(d, 8, 2, kb, vb, lens, seed=kb * 10 + vb), lens))


@pytest.mark.parametrize("pad,h_kv", [(24, 2), (8, 1), (56, 4)])
def test_padded_slot_stride(pad, h_kv):
    # slot_stride > slot_bytes: the padding rides along in the staged blocks (a 2-D
    # tensor box when a row of all heads is a multiple of 16 bytes, else a 1-D copy).
    tq = _tq()
    lens = [150, 16, 47]
    wl = _with_lens(_spec(128, 4 * h_kv, h_kv, 4, 2, lens, seed=pad), lens)
    pages, cb = gpu_append(tq, wl, slot_stride=wl.slot_bytes + pad, fill=0x77)
    out = gpu_decode(tq, wl, pages, cb)
    ref = _oracle_decode(wl, pages.cpu().numpy())
    assert decode_error(to_np_f64(out), ref) <= TOL


@pytest.mark.parametrize("q_dtype,out_dtype", [("float16", "float16"), ("float16", "float32"),
                                               ("float32", "float32"), ("bfloat16", "float32")])
def test_query_and_output_dtypes(q_dtype, out_dtype):
    tq = _tq()
    lens = [120, 40]
    wl = _with_lens(_spec(128, 16, 4, 4, 4, lens, seed=4), lens)
    wl.q = wl.q.float().to(getattr(torch, q_dtype))
    _case(tq, wl, out_dtype=getattr(torch, out_dtype))


def test_strided_query_and_output():
    # q and out as views with head and batch strides wider than the dense layout.
    tq = _tq()
    lens = [90, 200, 5]
    wl = _with_lens(_spec(64, 12, 3, 4, 3, lens, seed=8), lens)
    pages, cb = gpu_append(tq, wl)
    b, h, d = wl.q.shape
    qbig = torch.zeros(b, h, 2 * d, dtype=wl.q.dtype, device="cuda")
    qbig[..., d:] = wl.q.cuda()
    q = qbig[..., d:]
    obig = torch.full((b, 2 * h, d), float("nan"), dtype=torch.float32, device="cuda")
    out = obig[:, 1::2]
    assert q.stride(1) == 2 * d and out.stride(1) == 2 * d
    tq.paged_decode(out, q, pages, torch.from_numpy(wl.block_table).cuda(),
                    torch.from_numpy(wl.seq_lens).cuda(), cb, wl.spec.sign_seed, wl.spec.scale)
    torch.cuda.synchronize()
    assert torch.all(torch.isnan(obig[:, 0::2]))          # the other rows untouched
    ref = _oracle_decode(wl, pages.cpu().numpy())
    assert decode_error(to_np_f64(out), ref) <= TOL


@pytest.mark.parametrize("k_scale,v_scale", [(1.0, 1e18), (1.0, 1e-20), (1e-20, 1.0),
                                             (1e-12, 1e15)])
def test_extreme_key_and_value_magnitudes(k_scale, v_scale):
    # The decode reads norms from the slots: values of 1e18 or 1e-20 keep their weight
    # through the lazy softmax reference, keys of 1e-20 give uniform attention.
    tq = _tq()
    lens = [300, 64]
    wl = _with_lens(_spec(128, 8, 2, 4, 4, lens, dtype="float32", seed=12), lens)
    wl.k = wl.k * k_scale
    wl.v = wl.v * v_scale
    _case(tq, wl)


@pytest.mark.parametrize("kb,vb", [(4, 4), (3, 2), (8, 4)])
def test_gaussian_codebooks(kb, vb):
    tq = _tq()
    lens = [260, 31]
    wl = _with_lens(_spec(128, 16, 4, kb, vb, lens, seed=kb + vb), lens)
    pages, cb = gpu_append(tq, wl, kind="gauss")
    out = gpu_decode(tq, wl, pages, cb)
    ref = _oracle_decode(wl, pages.cpu().numpy(), kind="gauss")
    assert decode_error(to_np_f64(out), ref) <= TOL


def _hot_case(tq, wl, w, hot_lens, hot_dtype, seed, k_scale=3.0):
    """Append the workload, then decode with a hot window of w rows per sequence
    (hot_lens[b] of them in use) and compare with the oracle's joint softmax."""
    pages, cb = gpu_append(tq, wl)
    b, h_kv, d = wl.spec.batch, wl.spec.num_kv_heads, wl.spec.head_dim
    g = torch.Generator().manual_seed(seed)
    dt = getattr(torch, hot_dtype)
    hk = (torch.randn(b, w, h_kv, d, generator=g) * k_scale).to(dt)
    hv = torch.randn(b, w, h_kv, d, generator=g).to(dt)
    hl = np.asarray(hot_lens, dtype=np.int32)
    q = wl.q.cuda()
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    tq.paged_decode_hot(out, q, pages, torch.from_numpy(wl.block_table).cuda(),
                        torch.from_numpy(wl.seq_lens).cuda(), hk.cuda(), hv.cuda(),
                        torch.from_numpy(hl).cuda(), cb, wl.spec.sign_seed, wl.spec.scale)
    torch.cuda.synchronize()
    kt = oracle_table(d, wl.spec.k_bits)
    vt = oracle_table(d, wl.spec.v_bits)
    ref = O.paged_decode_hot(to_np_f64(wl.q), pages.cpu().numpy(), wl.block_table, wl.seq_lens,
                             to_np_f64(hk), to_np_f64(hv), hl, kt, vt, wl.spec.sign_seed,
                             wl.spec.scale)
    return to_np_f64(out), ref


@pytest.mark.parametrize("d,kb,vb,hot_dtype", [(128, 4, 4, "float16"), (64, 8, 2, "bfloat16"),
                                               (128, 3, 2, "float32"), (256, 4, 2, "float16")])
def test_hot_window_joins_the_softmax(d, kb, vb, hot_dtype):
    # sequences: long packed + full window, packed-empty + window only, packed only,
    # short packed + one hot token
    tq = _tq()
    lens = [300, 0, 17, 64]
    wl = _with_lens(_spec(d, 8, 2, kb, vb, lens, seed=d + kb), lens)
    got, ref = _hot_case(tq, wl, 24, [24, 5, 0, 1], hot_dtype, seed=kb)
    assert np.all(np.isfinite(got))
    assert decode_error(got, ref) <= TOL
    assert tq.get_device_error() == 0


def test_hot_window_dominant_and_long_split():
    # hot keys with larger norms than the packed ones carry most of the weight; the
    # packed part of the first sequence spans many CTAs
    tq = _tq()
    lens = [6000, 40, 0]
    wl = _with_lens(_spec(128, 16, 4, 4, 2, lens, seed=77), lens)
    got, ref = _hot_case(tq, wl, 64, [64, 64, 0], "float16", seed=5, k_scale=30.0)
    assert decode_error(got, ref) <= TOL
    assert np.all(got[2] == 0.0)                    # no tokens at all


def test_hot_window_bad_length_flagged():
    tq = _tq()
    lens = [50, 50]
    wl = _with_lens(_spec(128, 4, 1, 4, 4, lens, seed=3), lens)
    tq.get_device_error()
    got, _ = _hot_case(tq, wl, 8, [9, 3], "float16", seed=1)
    assert tq.get_device_error() & tq.DEVERR_SEQLEN_RANGE
    wl2 = _with_lens(_spec(128, 4, 1, 4, 4, lens, seed=3), lens)
    got2, ref2 = _hot_case(tq, wl2, 8, [0, 3], "float16", seed=1)
    assert decode_error(got[:1], ref2[:1]) <= TOL    # a bad length counts as 0 tokens
