"""Pins of the oracle's QJL residual sketch of the keys (tq-kv, "How It Works" step
[5]: SRHT QJL error correction; TorbuQuant, "Current Status": QJL residual)."""
import math
import os
import struct

import numpy as np
import pytest
import scipy.linalg

from oracle import gen_codebooks as G
from oracle import tq_oracle as O


def _table(d, bits):
    return G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(d, bits)))


def _bits_lsb_first(values, bits):
    out = bytearray((len(values) * bits + 7) // 8)
    for j, v in enumerate(values):
        for k in range(bits):
            if (int(v) >> k) & 1:
                p = j * bits + k
                out[p // 8] |= 1 << (p % 8)
    return bytes(out)


@pytest.mark.parametrize("d,bits", [(128, 3), (256, 2), (64, 4)])
def test_qjl_region_layout_by_hand(d, bits):
    rng = np.random.default_rng(d + bits)
    idx = rng.integers(0, 1 << bits, size=d)
    z = rng.integers(0, 2, size=d)
    norm, gamma = np.float32(3.25), np.float32(0.0625)
    raw = (_bits_lsb_first(idx, bits) + struct.pack("<f", norm) + _bits_lsb_first(z, 1)
           + struct.pack("<f", gamma))
    assert len(raw) == O.k_region_bytes(d, bits, True) == O.region_bytes(d, bits) + d // 8 + 4
    reg = O.encode_k_region_qjl(idx, norm, z, gamma, bits)
    assert bytes(reg) == raw
    gi, gn, gz, gg = O.decode_k_region_qjl(np.frombuffer(raw, np.uint8), d, bits)
    np.testing.assert_array_equal(gi, idx)
    np.testing.assert_array_equal(gz, z)
    assert gn == norm and gg == gamma


def test_qjl_score_identity_with_explicit_matrices():
    # <q, k_hat> = n (<R q, c> + gamma sqrt(pi/2)/sqrt(D) <S R q, 2z - 1>) with R and S
    # built as explicit matrices from scipy's Hadamard and the sign vectors.
    d, bits = 128, 2
    t = _table(d, bits)
    s1, s2 = O.rht_signs(d, 3), O.rht_signs(d, 11)
    r_mat = scipy.linalg.hadamard(d) * s1[None, :] / math.sqrt(d)
    s_mat = scipy.linalg.hadamard(d) * s2[None, :] / math.sqrt(d)
    rng = np.random.default_rng(0)
    x = rng.standard_normal((20, d)) * 2.0
    q = rng.standard_normal((5, d))
    idx, n, z, g, u, _ = O.quantize_keys_qjl(x, s1, t, s2)
    c = t.centroids.astype(np.float64)[idx]
    np.testing.assert_allclose(g, np.linalg.norm(u - c, axis=1), rtol=1e-6)
    np.testing.assert_array_equal(z, ((u - c) @ s_mat.T >= 0).astype(np.int64))
    khat = O.dequantize_keys_qjl(idx, n, z, g, t, s1, s2)
    for qq in q:
        qr = r_mat @ qq
        ref = n.astype(np.float64) * (c @ qr + g.astype(np.float64) * math.sqrt(math.pi / 2)
                                      / math.sqrt(d) * ((2 * z - 1) @ (s_mat @ qr)))
        np.testing.assert_allclose(khat @ qq, ref, rtol=1e-10, atol=1e-10)


def test_qjl_estimator_is_unbiased_over_sketch_signs():
    # For fixed y and r, the average of gamma sqrt(pi/2)/sqrt(D) <S y, sign(S r)> over
    # independent sketch signs approaches <y, r> (the Gaussian-sketch constant; the
    # randomized Hadamard rows are near-Gaussian at D = 128).
    d = 128
    rng = np.random.default_rng(5)
    y = rng.standard_normal(d)
    r = 0.3 * rng.standard_normal(d) + 0.2 * y        # correlated with y
    est = []
    for seed in range(4000):
        s2 = O.rht_signs(d, 1000 + seed)
        z, gamma = O.qjl_sketch(r, s2)
        est.append(float(y @ O.qjl_correction(z, gamma, s2)))
    est = np.array(est)
    true = float(y @ r)
    sem = est.std() / math.sqrt(len(est))
    assert abs(est.mean() - true) < 4 * sem + 0.01 * abs(true), (est.mean(), true, sem)
    # the uncorrected (MSE-only) estimate of <y, r> is 0: the correction carries the signal
    assert abs(true) > 10 * sem


def test_quantize_append_qjl_slot_placement():
    d, h_kv = 64, 2
    kt, vt = _table(d, 3), _table(d, 2)
    kb, vb = O.k_region_bytes(d, 3, True), O.region_bytes(d, 2)
    pages = np.full((2, 16, h_kv, kb + vb + 8), 0xA5, dtype=np.uint8)
    rng = np.random.default_rng(2)
    k = rng.standard_normal((3, h_kv, d))
    v = rng.standard_normal((3, h_kv, d))
    out = O.quantize_append_qjl(pages, np.array([5, -1, 17]), k, v, kt, vt, 0, 9)
    for tok, slot in ((0, 5), (2, 17)):
        for h in range(h_kv):
            idx, n, z, g, _, _ = O.quantize_keys_qjl(k[tok, h], O.rht_signs(d, 0), kt,
                                                     O.rht_signs(d, 9))
            vi, vn, _, _ = O.quantize_rows(v[tok, h], O.rht_signs(d, 0), vt)
            region = out[slot // 16, slot % 16, h]
            assert bytes(region[:kb]) == bytes(O.encode_k_region_qjl(idx, n, z, g, 3))
            assert bytes(region[kb:kb + vb]) == bytes(O.encode_region(vi, vn, 2))
            assert np.all(region[kb + vb:] == 0xA5)
    assert np.all(out[0, 6:] == 0xA5) and np.all(out[1, :1] == 0xA5)


def test_qjl_decode_brute_force():
    d, h_q, h_kv = 64, 4, 2
    kt, vt = _table(d, 2), _table(d, 2)
    lens = [21, 3]
    rng = np.random.default_rng(8)
    kb, vb = O.k_region_bytes(d, 2, True), O.region_bytes(d, 2)
    pages = np.zeros((3, 16, h_kv, kb + vb), dtype=np.uint8)
    bt = np.array([[0, 2], [1, 0]])
    for b, n in enumerate(lens):
        slots = bt[b, np.arange(n) // 16] * 16 + np.arange(n) % 16
        pages = O.quantize_append_qjl(pages, slots, rng.standard_normal((n, h_kv, d)),
                                      rng.standard_normal((n, h_kv, d)), kt, vt, 4, 6)
    q = rng.standard_normal((2, h_q, d))
    got = O.paged_decode_qjl(q, pages, bt, np.array(lens), kt, vt, 4, 6, 0.125)
    s1, s2 = O.rht_signs(d, 4), O.rht_signs(d, 6)
    r_mat = scipy.linalg.hadamard(d) * s1[None, :] / math.sqrt(d)
    s_mat = scipy.linalg.hadamard(d) * s2[None, :] / math.sqrt(d)
    for b, n in enumerate(lens):
        for h in range(h_q):
            kv = h // 2
            sc, vals = [], []
            for t in range(n):
                slot = pages[bt[b, t // 16], t % 16, kv]
                ki, kn, kz, kg = O.decode_k_region_qjl(slot[:kb], d, 2)
                vi, vn = O.decode_region(slot[kb:kb + vb], d, 2)
                qr = r_mat @ q[b, h]
                score = float(kn) * (kt.centroids.astype(np.float64)[ki] @ qr + float(kg)
                                     * math.sqrt(math.pi / 2) / math.sqrt(d)
                                     * ((2 * kz - 1) @ (s_mat @ qr)))
                sc.append(0.125 * score)
                vals.append(float(vn) * (r_mat.T @ vt.centroids.astype(np.float64)[vi]))
            mx = max(sc)
            w = [math.exp(x - mx) for x in sc]
            ref = sum(wi * vv for wi, vv in zip(w, vals)) / sum(w)
            np.testing.assert_allclose(got[b, h], ref, rtol=0, atol=1e-10)
