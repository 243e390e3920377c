"""GPU parity of the dense-rotation variant (tcgen05 append, dense decode) against the
oracle with the same rotation table (R = hi + lo of the seeded Haar matrix)."""
import numpy as np
import pytest
import torch

from oracle import tq_oracle as O
from oracle import gen_rotations as GR
from kv_cache_vector_append_b200 import workloads as W
from tests.gpu_helpers import decode_error, oracle_table, require_gpu, to_np_f64
import os

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _tq():
    require_gpu()
    import kv_cache_vector_append_b200 as tq
    return tq


def _rot(d):
    dim, seed, hi, lo = GR.read_table(os.path.join(GR.DEFAULT_OUT, GR.table_filename(d)))
    rot = O.dense_rotation(dim, seed)
    np.testing.assert_array_equal(rot.hi, hi)
    return rot


def _spec(d, h_q, h_kv, kb, vb, seq, batch, seed, dtype="bfloat16"):
    return W.WorkloadSpec(f"dense-d{d}", d, h_q, h_kv, batch, kb, vb, dtype, seq_len=seq,
                          n_outliers=2, outlier_factor=20.0, seed=seed)


def _append(tq, wl, slot_mapping=None, fill=0):
    pages = W.empty_pages(wl, device="cuda", fill=fill)
    sm = wl.slot_mapping if slot_mapping is None else slot_mapping
    cb = tq.load_codebooks(wl.spec.head_dim, wl.spec.k_bits, wl.spec.v_bits, "cuda")
    rot = tq.load_rotation(wl.spec.head_dim, "cuda")
    tq.quantize_append_dense(pages, torch.from_numpy(np.ascontiguousarray(sm)).cuda(),
                             wl.k.cuda(), wl.v.cuda(), cb, rot)
    torch.cuda.synchronize()
    return pages, cb, rot


def _regions(pages_np, wl, kind):
    d = wl.spec.head_dim
    kb, vb = O.region_bytes(d, wl.spec.k_bits), O.region_bytes(d, wl.spec.v_bits)
    s = wl.slot_mapping
    rows = pages_np[s // 16, s % 16]
    return rows[..., :kb] if kind == 0 else rows[..., kb:kb + vb]


def _check_append(tq, wl):
    pages, cb, rot = _append(tq, wl)
    p = pages.cpu().numpy()
    d = wl.spec.head_dim
    orot = _rot(d)
    mism = total = 0
    for kind, (src, bits) in enumerate(((wl.k, wl.spec.k_bits), (wl.v, wl.spec.v_bits))):
        t = oracle_table(d, bits)
        # bit exact on the kernel's own unit coordinates
        x = src.reshape(-1, d).cuda()
        u = torch.empty(x.shape, dtype=torch.float32, device="cuda")
        n = torch.empty(x.shape[0], dtype=torch.float32, device="cuda")
        tq.rotate_unit_dense(u, n, x, rot)
        idx = O.encode(u.cpu().numpy().astype(np.float64), t.boundaries)
        expect = O.encode_region(idx, n.cpu().numpy(), bits).reshape(src.shape[0], src.shape[1], -1)
        got = _regions(p, wl, kind)
        bad_rows = np.nonzero(np.any(got != expect, axis=-1))[0]
        assert bad_rows.size == 0, f"kind {kind}: {bad_rows.size} rows differ"
        # end to end against the fp64 oracle with the same rotation
        ri, rn, ru, _ = O.quantize_rows(to_np_f64(src), orot, t)
        gi, gn = O.decode_region(got, d, bits)
        np.testing.assert_allclose(gn, rn, rtol=1e-6, atol=0)
        bad = gi != ri
        mism += int(bad.sum())
        total += bad.size
        if bad.any():
            b = t.boundaries.astype(np.float64)
            assert np.all(np.min(np.abs(ru[bad][:, None] - b[None, :]), axis=1) < 1e-5)
    assert mism <= 1e-4 * total, f"{mism} of {total} codes differ"
    return pages, cb, rot


@pytest.mark.parametrize("d,h_kv,kb,vb", [(128, 8, 4, 4), (128, 4, 4, 2), (64, 2, 8, 8),
                                          (128, 1, 3, 2), (64, 16, 2, 4), (128, 8, 8, 8)])
def test_dense_append_bit_exact_and_end_to_end(d, h_kv, kb, vb):
    tq = _tq()
    # 3 sequences of 77 tokens: several tiles of 128 pairs and a ragged last tile
    _check_append(tq, W.generate(_spec(d, h_kv, h_kv, kb, vb, 77, 3, seed=d + kb)))


def test_dense_append_extreme_rows():
    # rows far from unit scale take the rescaled CUDA-core path of the same kernel
    tq = _tq()
    wl = W.generate(_spec(128, 4, 4, 4, 4, 40, 2, seed=3))
    f = torch.tensor([[1.0, 1e-20, 1e18, 1.0, 1e-30, 1e30][t % 6] for t in range(wl.k.shape[0])],
                     dtype=torch.float64)[:, None, None]
    wl.k = (wl.k.double() * f).to(torch.bfloat16)
    wl.v = (wl.v.double() * f).to(torch.bfloat16)
    _check_append(tq, wl)


@pytest.mark.parametrize("d,h_q,h_kv,kb,vb", [(128, 32, 8, 4, 4), (128, 28, 4, 4, 2),
                                              (64, 14, 2, 8, 8), (128, 16, 2, 3, 2)])
def test_dense_decode(d, h_q, h_kv, kb, vb):
    tq = _tq()
    lens = [300, 17, 64, 0]
    spec = _spec(d, h_q, h_kv, kb, vb, max(lens), len(lens), seed=h_q)
    wl = W.generate(spec)
    wl.seq_lens = np.asarray(lens, dtype=np.int32)
    pages, cb, rot = _check_append(tq, wl)
    q = wl.q.cuda()
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    tq.paged_decode_dense(out, q, pages, torch.from_numpy(wl.block_table).cuda(),
                          torch.from_numpy(wl.seq_lens).cuda(), cb, rot, spec.scale)
    torch.cuda.synchronize()
    ref = O.paged_decode(to_np_f64(wl.q), pages.cpu().numpy(), wl.block_table, wl.seq_lens,
                         oracle_table(d, kb), oracle_table(d, vb), 0, spec.scale,
                         rotation=_rot(d))
    got = to_np_f64(out)
    assert np.all(got[3] == 0.0)
    assert decode_error(got, ref) <= TOL
    assert tq.get_device_error() == 0


def test_dense_full_size_layer_sampled():
    # The Llama-3-8B-shaped layer (8 KV heads, D = 128, 4-bit K and V) at 8 x 8192
    # tokens in the launch shape the dense path uses; sampled tokens against the oracle.
    tq = _tq()
    wl = W.generate(W.CONFIGS[2].scaled(batch=8))
    pages, cb, rot = _append(tq, wl)
    p = pages.cpu().numpy()
    rng = np.random.default_rng(2)
    toks = np.sort(rng.choice(wl.k.shape[0], size=2000, replace=False))
    orot = _rot(128)
    mism = total = 0
    for kind, (src, bits) in enumerate(((wl.k, 4), (wl.v, 4))):
        t = oracle_table(128, bits)
        ri, rn, ru, _ = O.quantize_rows(to_np_f64(src[torch.from_numpy(toks)]), orot, t)
        s = wl.slot_mapping[toks]
        rows = p[s // 16, s % 16]
        kb = O.region_bytes(128, 4)
        reg = rows[..., :kb] if kind == 0 else rows[..., kb:2 * kb]
        gi, gn = O.decode_region(reg, 128, bits)
        np.testing.assert_allclose(gn, rn, rtol=1e-6, atol=0)
        mism += int((gi != ri).sum())
        total += gi.size
    assert mism <= 1e-4 * total
    out = torch.empty(wl.q.shape, dtype=torch.float32, device="cuda")
    tq.paged_decode_dense(out, wl.q.cuda(), pages, torch.from_numpy(wl.block_table).cuda(),
                          torch.from_numpy(wl.seq_lens).cuda(), cb, rot, wl.spec.scale)
    torch.cuda.synchronize()
    seqs = np.array([0, 5])
    ref = O.paged_decode(to_np_f64(wl.q)[seqs], p, wl.block_table[seqs], wl.seq_lens[seqs],
                         oracle_table(128, 4), oracle_table(128, 4), 0, wl.spec.scale,
                         rotation=orot)
    assert decode_error(to_np_f64(out)[seqs], ref) <= TOL


def test_dense_unsupported_geometries():
    tq = _tq()
    from kv_cache_vector_append_b200 import _binding as B
    wl = W.generate(_spec(128, 3, 3, 4, 4, 20, 1, seed=1))      # 3 heads: no tensor box
    with pytest.raises(B.TQError) as e:
        _append(tq, wl)
    assert e.value.status == B.ERR_UNSUPPORTED
    wl = W.generate(_spec(256, 2, 2, 4, 4, 20, 1, seed=1))      # D = 256: not built
    pages = W.empty_pages(wl, device="cuda")
    cb = tq.load_codebooks(256, 4, 4, "cuda")
    rot = tq.load_rotation(256, "cuda")
    with pytest.raises(B.TQError) as e:
        tq.quantize_append_dense(pages, torch.from_numpy(wl.slot_mapping).cuda(), wl.k.cuda(),
                                 wl.v.cuda(), cb, rot)
    assert e.value.status == B.ERR_UNSUPPORTED
