"""Pins of the oracle's paged decode attention."""
import math
import os

import numpy as np
import pytest
import scipy.linalg

from oracle import tq_oracle as O
from oracle import gen_codebooks as G


def _table(d, bits):
    return G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(d, bits)))


def _make_cache(d, h_kv, lens, kbits, vbits, seed=0, bs=16, sign_seed=0, perm=True):
    rng = np.random.default_rng(seed)
    kt, vt = _table(d, kbits), _table(d, vbits)
    nblk_seq = [(n + bs - 1) // bs for n in lens]
    pool = max(1, sum(nblk_seq))
    order = rng.permutation(pool) if perm else np.arange(pool)
    max_blocks = max(1, max(nblk_seq))
    bt = np.zeros((len(lens), max_blocks), dtype=np.int64)
    pos = 0
    for b, nb in enumerate(nblk_seq):
        bt[b, :nb] = order[pos:pos + nb]
        pos += nb
    sb = O.slot_bytes(d, kbits, vbits)
    pages = np.zeros((pool, bs, h_kv, sb), dtype=np.uint8)
    for b, n in enumerate(lens):
        if n == 0:
            continue
        k = rng.standard_normal((n, h_kv, d)) * rng.lognormal(0, 0.5, size=(1, h_kv, d))
        v = rng.standard_normal((n, h_kv, d))
        slots = bt[b, np.arange(n) // bs] * bs + np.arange(n) % bs
        pages = O.quantize_append(pages, slots, k, v, kt, vt, sign_seed)
    return pages, bt, np.array(lens), kt, vt


def _brute_force(q, pages, bt, lens, kt, vt, sign_seed, scale):
    # Explicit rotation matrix from the library Hadamard, python loops, math.exp.
    bsz, h_q, d = q.shape
    bs, h_kv = pages.shape[1], pages.shape[2]
    g = h_q // h_kv
    s = O.rht_signs(d, sign_seed)
    r = scipy.linalg.hadamard(d) * s[None, :] / math.sqrt(d)
    kb, vb = O.region_bytes(d, kt.bits), O.region_bytes(d, vt.bits)
    out = np.zeros_like(q, dtype=np.float64)
    for b in range(bsz):
        for h in range(h_q):
            kv = h // g
            keys, vals = [], []
            for t in range(int(lens[b])):
                slot = pages[bt[b, t // bs], t % bs, kv]
                ki, kn = O.decode_region(slot[:kb], d, kt.bits)
                vi, vn = O.decode_region(slot[kb:kb + vb], d, vt.bits)
                keys.append(float(kn) * (r.T @ kt.centroids.astype(np.float64)[ki]))
                vals.append(float(vn) * (r.T @ vt.centroids.astype(np.float64)[vi]))
            if not keys:
                continue
            sc = [scale * float(np.dot(q[b, h], k_)) for k_ in keys]
            mx = max(sc)
            w = [math.exp(x - mx) for x in sc]
            tot = sum(w)
            out[b, h] = sum(wi * v_ for wi, v_ in zip(w, vals)) / tot
    return out


@pytest.mark.parametrize("d,h_q,h_kv,kbits,vbits", [(64, 4, 2, 8, 8), (128, 7, 1, 4, 2),
                                                    (128, 4, 4, 3, 2)])
def test_decode_brute_force(d, h_q, h_kv, kbits, vbits):
    lens = [1, 17, 33, 0]
    pages, bt, sl, kt, vt = _make_cache(d, h_kv, lens, kbits, vbits, seed=d + h_q)
    q = np.random.default_rng(1).standard_normal((len(lens), h_q, d))
    scale = 1 / math.sqrt(d)
    ref = _brute_force(q, pages, bt, sl, kt, vt, 0, scale)
    got = O.paged_decode(q, pages, bt, sl, kt, vt, 0, scale)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    rot = O.paged_decode_rotated(q, pages, bt, sl, kt, vt, 0, scale, split_tokens=16)
    np.testing.assert_allclose(rot, ref, rtol=0, atol=1e-12)
    assert np.all(got[3] == 0.0)


def test_rotated_domain_and_split_merge_equal_plain():
    d, h_kv, h_q = 128, 2, 8
    lens = [200, 64, 5]
    pages, bt, sl, kt, vt = _make_cache(d, h_kv, lens, 4, 4, seed=7)
    q = np.random.default_rng(2).standard_normal((3, h_q, d)) * 2
    scale = 1 / math.sqrt(d)
    ref = O.paged_decode(q, pages, bt, sl, kt, vt, 0, scale)
    for split in (0, 16, 48, 160):
        got = O.paged_decode_rotated(q, pages, bt, sl, kt, vt, 0, scale, split_tokens=split)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_single_token_returns_its_value():
    d = 64
    pages, bt, sl, kt, vt = _make_cache(d, 1, [1], 8, 8, seed=3)
    q = np.random.default_rng(0).standard_normal((1, 3, d))
    out = O.paged_decode(q, pages, bt, sl, kt, vt, 0, 0.125)
    slot = pages[bt[0, 0], 0, 0]
    vi, vn = O.decode_region(slot[O.region_bytes(d, 8):], d, 8)
    vhat = O.dequantize_rows(vi, vn, vt, O.rht_signs(d, 0))
    for h in range(3):
        np.testing.assert_allclose(out[0, h], vhat, atol=1e-13)


def test_equal_scores_average_values():
    # Identical keys -> uniform weights -> output is the mean of the values.
    d, bs = 64, 16
    kt, vt = _table(d, 4), _table(d, 4)
    n = 20
    rng = np.random.default_rng(4)
    kk = np.repeat(rng.standard_normal((1, 1, d)), n, axis=0)
    vv = rng.standard_normal((n, 1, d))
    pages = np.zeros((2, bs, 1, O.slot_bytes(d, 4, 4)), dtype=np.uint8)
    pages = O.quantize_append(pages, np.arange(n), kk, vv, kt, vt, 0)
    bt = np.array([[0, 1]])
    out = O.paged_decode(rng.standard_normal((1, 1, d)), pages, bt, np.array([n]), kt, vt, 0, 1.0)
    s = O.rht_signs(d, 0)
    vhat = []
    for t in range(n):
        vi, vn = O.decode_region(pages[t // bs, t % bs, 0, O.region_bytes(d, 4):], d, 4)
        vhat.append(O.dequantize_rows(vi, vn, vt, s))
    np.testing.assert_allclose(out[0, 0], np.mean(vhat, axis=0), atol=1e-13)


def test_gqa_grouping_is_contiguous():
    # Query heads 0..G-1 read KV head 0, heads G..2G-1 read KV head 1.
    d, g = 64, 3
    pages, bt, sl, kt, vt = _make_cache(d, 2, [9], 8, 8, seed=5)
    q = np.random.default_rng(6).standard_normal((1, 2 * g, d))
    out = O.paged_decode(q, pages, bt, sl, kt, vt, 0, 0.125)
    for h in range(2 * g):
        kv = h // g
        single = O.paged_decode(q[:, h:h + 1], pages[:, :, kv:kv + 1], bt, sl, kt, vt, 0, 0.125)
        np.testing.assert_allclose(out[:, h], single[:, 0], atol=1e-14)


def _hot_window(bsz, w, h_kv, d, seed, dtype=np.float16):
    rng = np.random.default_rng(seed)
    hk = (rng.standard_normal((bsz, w, h_kv, d)) * 1.5).astype(dtype)
    hv = rng.standard_normal((bsz, w, h_kv, d)).astype(dtype)
    return hk, hv


def test_hot_window_empty_equals_paged_decode():
    d, h_kv, h_q = 64, 2, 6
    lens = [40, 1, 0]
    pages, bt, sl, kt, vt = _make_cache(d, h_kv, lens, 4, 2, seed=9)
    q = np.random.default_rng(3).standard_normal((3, h_q, d))
    hk, hv = _hot_window(3, 5, h_kv, d, 1)
    got = O.paged_decode_hot(q, pages, bt, sl, hk, hv, np.zeros(3, int), kt, vt, 0, 0.125)
    ref = O.paged_decode(q, pages, bt, sl, kt, vt, 0, 0.125)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-14)


def test_hot_window_only_is_plain_attention():
    # No packed tokens: textbook softmax attention over the fp16 rows, by loops.
    d, h_kv, h_q, w = 64, 2, 4, 7
    pages, bt, sl, kt, vt = _make_cache(d, h_kv, [0, 0], 4, 4, seed=2)
    q = np.random.default_rng(5).standard_normal((2, h_q, d))
    hk, hv = _hot_window(2, w, h_kv, d, 6)
    hl = np.array([w, 3])
    got = O.paged_decode_hot(q, pages, bt, sl, hk, hv, hl, kt, vt, 0, 0.125)
    for b in range(2):
        for h in range(h_q):
            kv = h // (h_q // h_kv)
            sc = [0.125 * sum(float(q[b, h, j]) * float(hk[b, t, kv, j]) for j in range(d))
                  for t in range(hl[b])]
            mx = max(sc)
            e = [math.exp(x - mx) for x in sc]
            ref = sum(ei * hv[b, t, kv].astype(np.float64) for t, ei in enumerate(e)) / sum(e)
            np.testing.assert_allclose(got[b, h], ref, rtol=0, atol=1e-12)
    assert np.all(O.paged_decode_hot(q, pages, bt, sl, hk, hv, np.zeros(2, int), kt, vt, 0,
                                     0.125) == 0.0)


def test_hot_window_joins_the_packed_softmax():
    # One softmax over packed and hot tokens: brute force over the concatenated rows
    # (packed rows dequantized through an explicit rotation matrix).
    d, h_kv, h_q = 64, 1, 3
    lens = [20, 33]
    pages, bt, sl, kt, vt = _make_cache(d, h_kv, lens, 3, 2, seed=4)
    q = np.random.default_rng(8).standard_normal((2, h_q, d)) * 2
    hk, hv = _hot_window(2, 6, h_kv, d, 9)
    hl = np.array([6, 2])
    got = O.paged_decode_hot(q, pages, bt, sl, hk, hv, hl, kt, vt, 0, 0.125)
    s = O.rht_signs(d, 0)
    r = scipy.linalg.hadamard(d) * s[None, :] / math.sqrt(d)
    kb, vb = O.region_bytes(d, 3), O.region_bytes(d, 2)
    for b in range(2):
        keys, vals = [], []
        for t in range(lens[b]):
            slot = pages[bt[b, t // 16], t % 16, 0]
            ki, kn = O.decode_region(slot[:kb], d, 3)
            vi, vn = O.decode_region(slot[kb:kb + vb], d, 2)
            keys.append(float(kn) * (r.T @ kt.centroids.astype(np.float64)[ki]))
            vals.append(float(vn) * (r.T @ vt.centroids.astype(np.float64)[vi]))
        keys += [hk[b, t, 0].astype(np.float64) for t in range(hl[b])]
        vals += [hv[b, t, 0].astype(np.float64) for t in range(hl[b])]
        for h in range(h_q):
            sc = [0.125 * float(np.dot(q[b, h], k_)) for k_ in keys]
            mx = max(sc)
            e = [math.exp(x - mx) for x in sc]
            ref = sum(ei * v_ for ei, v_ in zip(e, vals)) / sum(e)
            np.testing.assert_allclose(got[b, h], ref, rtol=0, atol=1e-12)
    # and the split-KV merge of the packed part with the hot part equals it too
    for b in range(2):
        slots = O.gather_sequence(pages, bt[b], lens[b])
        ki, kn = O.decode_region(slots[..., :kb], d, 3)
        vi, vn = O.decode_region(slots[..., kb:kb + vb], d, 2)
        for h in range(h_q):
            qr = O.rht_forward(q[b, h], s)
            m1, l1, o1 = O.rotated_domain_partial(qr, ki[:, 0], kn[:, 0], vi[:, 0], vn[:, 0], kt,
                                                  vt, 0.125)
            o1 = O.rht_inverse(o1, s)
            sh = 0.125 * (hk[b, :hl[b], 0].astype(np.float64) @ q[b, h])
            m2 = np.max(sh)
            e2 = np.exp(sh - m2)
            o2 = e2 @ hv[b, :hl[b], 0].astype(np.float64)
            merged = O.merge_partials([(m1, l1, o1), (m2, np.sum(e2), o2)])
            np.testing.assert_allclose(merged, got[b, h], rtol=0, atol=1e-12)
