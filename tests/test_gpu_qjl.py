"""GPU parity of the QJL residual sketch of the keys (tq_quantize_append_qjl,
tq_paged_decode_qjl) against the oracle."""
import numpy as np
import pytest
import torch

from oracle import tq_oracle as O
from kv_cache_vector_append_b200 import workloads as W
from tests.gpu_helpers import decode_error, oracle_table, require_gpu, to_np_f64

pytestmark = pytest.mark.gpu
TOL = 2e-3
QJL_SEED = 77


def _tq():
    require_gpu()
    import kv_cache_vector_append_b200 as tq
    return tq


def _spec(d, h_q, h_kv, kb, vb, seq, batch, seed, dtype="bfloat16"):
    return W.WorkloadSpec(f"qjl-d{d}", d, h_q, h_kv, batch, kb, vb, dtype, seq_len=seq,
                          n_outliers=2, outlier_factor=20.0, seed=seed)


def _append(tq, wl):
    d = wl.spec.head_dim
    sb = tq.slot_bytes_qjl(d, wl.spec.k_bits, wl.spec.v_bits)
    assert sb == O.k_region_bytes(d, wl.spec.k_bits, True) + O.region_bytes(d, wl.spec.v_bits)
    # slot_stride: the slot bytes rounded up to a multiple of 8 (the padding is never written)
    pages = W.empty_pages(wl, device="cuda", slot_stride=(sb + 7) // 8 * 8)
    cb = tq.load_codebooks(d, wl.spec.k_bits, wl.spec.v_bits, "cuda")
    tq.quantize_append_qjl(pages, torch.from_numpy(wl.slot_mapping).cuda(), wl.k.cuda(),
                           wl.v.cuda(), cb, wl.spec.sign_seed, QJL_SEED)
    torch.cuda.synchronize()
    return pages, cb


def _check_append(tq, wl):
    pages, cb = _append(tq, wl)
    p = pages.cpu().numpy()
    d, kbits, vbits = wl.spec.head_dim, wl.spec.k_bits, wl.spec.v_bits
    kt, vt = oracle_table(d, kbits), oracle_table(d, vbits)
    s1, s2 = O.rht_signs(d, wl.spec.sign_seed), O.rht_signs(d, QJL_SEED)
    kb = O.k_region_bytes(d, kbits, True)
    vb = O.region_bytes(d, vbits)
    rows = p[wl.slot_mapping // 16, wl.slot_mapping % 16]          # [T, H_kv, slot]
    gi, gn, gz, gg = O.decode_k_region_qjl(rows[..., :kb], d, kbits)
    ri, rn, rz, rg, ru, _ = O.quantize_keys_qjl(to_np_f64(wl.k), s1, kt, s2)
    # codes and norms: the end-to-end bar of the plain append
    np.testing.assert_allclose(gn, rn, rtol=1e-6, atol=0)
    bad = gi != ri
    assert bad.sum() <= 1e-4 * bad.size, f"{bad.sum()} of {bad.size} codes differ"
    if bad.any():
        b = kt.boundaries.astype(np.float64)
        assert np.all(np.min(np.abs(ru[bad][:, None] - b[None, :]), axis=1) < 1e-5)
    # the sketch, on rows whose codes all match (a flipped code changes the residual)
    same = ~np.any(bad, axis=-1)
    np.testing.assert_allclose(gg[same], rg[same], rtol=1e-5, atol=1e-7)
    c = kt.centroids.astype(np.float64)[ri]
    sr = O.rht_forward(ru - c, s2)                                   # oracle S r, fp64
    zbad = (gz != rz) & same[..., None]
    near = np.abs(sr) < 1e-4 * np.maximum(rg.astype(np.float64), 1e-30)[..., None]
    assert np.all(near[zbad]), f"{zbad.sum()} sketch bits differ away from 0"
    assert zbad.sum() <= 1e-3 * zbad.size
    # the V region is the plain one
    vi, vn = O.decode_region(rows[..., kb:kb + vb], d, vbits)
    rvi, rvn, _, _ = O.quantize_rows(to_np_f64(wl.v), s1, vt)
    np.testing.assert_allclose(vn, rvn, rtol=1e-6, atol=0)
    assert (vi != rvi).sum() <= 1e-4 * vi.size
    return pages, cb


@pytest.mark.parametrize("d,h_q,h_kv,kb,vb", [(128, 32, 8, 4, 4), (128, 28, 4, 3, 2),
                                              (256, 16, 2, 2, 4), (128, 8, 8, 2, 2),
                                              (256, 8, 1, 4, 8)])
def test_qjl_append_and_decode(d, h_q, h_kv, kb, vb):
    tq = _tq()
    lens = [200, 17, 33, 0]
    spec = _spec(d, h_q, h_kv, kb, vb, max(lens), len(lens), seed=d + kb + vb)
    wl = W.generate(spec)
    pages, cb = _check_append(tq, wl)
    wl.seq_lens = np.asarray(lens, dtype=np.int32)
    q = wl.q.cuda()
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    tq.paged_decode_qjl(out, q, pages, torch.from_numpy(wl.block_table).cuda(),
                        torch.from_numpy(wl.seq_lens).cuda(), cb, spec.sign_seed, QJL_SEED,
                        spec.scale)
    torch.cuda.synchronize()
    ref = O.paged_decode_qjl(to_np_f64(wl.q), pages.cpu().numpy(), wl.block_table, wl.seq_lens,
                             oracle_table(d, kb), oracle_table(d, vb), spec.sign_seed, QJL_SEED,
                             spec.scale)
    got = to_np_f64(out)
    assert np.all(got[3] == 0.0)
    assert decode_error(got, ref) <= TOL
    assert tq.get_device_error() == 0


def test_qjl_full_size_layer_sampled():
    # Llama-3-8B-shaped layer with 3-bit keys and the sketch, 4 x 8192 tokens
    tq = _tq()
    spec = W.CONFIGS[2].scaled(batch=4, k_bits=3, v_bits=2)
    wl = W.generate(spec)
    pages, cb = _append(tq, wl)
    out = torch.empty(wl.q.shape, dtype=torch.float32, device="cuda")
    tq.paged_decode_qjl(out, wl.q.cuda(), pages, torch.from_numpy(wl.block_table).cuda(),
                        torch.from_numpy(wl.seq_lens).cuda(), cb, spec.sign_seed, QJL_SEED,
                        spec.scale)
    torch.cuda.synchronize()
    seqs = np.array([1])
    ref = O.paged_decode_qjl(to_np_f64(wl.q)[seqs], pages.cpu().numpy(), wl.block_table[seqs],
                             wl.seq_lens[seqs], oracle_table(128, 3), oracle_table(128, 2),
                             spec.sign_seed, QJL_SEED, spec.scale)
    assert decode_error(to_np_f64(out)[seqs], ref) <= TOL


def test_qjl_unsupported():
    tq = _tq()
    from kv_cache_vector_append_b200 import _binding as B
    wl = W.generate(_spec(64, 4, 2, 4, 4, 20, 1, seed=1))
    pages = W.empty_pages(wl, device="cuda", slot_stride=(tq.slot_bytes_qjl(64, 4, 4) + 7) // 8 * 8)
    cb = tq.load_codebooks(64, 4, 4, "cuda")
    with pytest.raises(B.TQError) as e:
        tq.quantize_append_qjl(pages, torch.from_numpy(wl.slot_mapping).cuda(), wl.k.cuda(),
                               wl.v.cuda(), cb, 0, QJL_SEED)
    assert e.value.status == B.ERR_UNSUPPORTED
