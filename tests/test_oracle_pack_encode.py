"""Pins of the oracle's slot layout, bit packing, encode and slot writes."""
import math
import os
import struct

import numpy as np
import pytest

from oracle import tq_oracle as O
from oracle import gen_codebooks as G


def _table(d, bits):
    return G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(d, bits)))


def test_slot_formula_and_printed_ratios(golden):
    for row in golden("slot_layout.txt"):
        if row[0] == "slot":
            d, kb, vb, k, v, sb = map(int, row[1:])
            assert O.region_bytes(d, kb) == k
            assert O.region_bytes(d, vb) == v
            assert O.slot_bytes(d, kb, vb) == sb
        else:
            d, bits, base, printed = int(row[1]), int(row[2]), int(row[3]), float(row[4])
            assert round(base / O.region_bytes(d, bits), 1) == printed


def test_slot_position():
    # The diagram's example slot 17 with block_size 16: block 1, row 1.
    assert O.slot_position(17, 16) == (1, 1)
    assert O.slot_position(15, 16) == (0, 15)
    assert O.slot_position(16, 16) == (1, 0)


@pytest.mark.parametrize("bits", range(1, 9))
@pytest.mark.parametrize("d", [64, 128, 256])
def test_pack_single_index_brute_force(bits, d):
    # Every value at every position sets exactly the bits j*b + k where value has bit k.
    nbytes = (d * bits + 7) // 8
    values = np.arange(1, 1 << bits)
    for j in range(d):
        idx = np.zeros((values.size, d), dtype=np.int64)
        idx[:, j] = values
        packed = O.pack_bits(idx, bits)
        assert packed.shape == (values.size, nbytes)
        for r, val in enumerate(values):
            expect = np.zeros(nbytes * 8, dtype=np.uint8)
            for k in range(bits):
                expect[j * bits + k] = (val >> k) & 1
            got = np.unpackbits(packed[r], bitorder="little")
            np.testing.assert_array_equal(got, expect)
        np.testing.assert_array_equal(O.unpack_bits(packed, d, bits), idx)


@pytest.mark.parametrize("bits", range(1, 9))
def test_pack_roundtrip_random(bits):
    rng = np.random.default_rng(bits)
    idx = rng.integers(0, 1 << bits, size=(50, 128))
    np.testing.assert_array_equal(O.unpack_bits(O.pack_bits(idx, bits), 128, bits), idx)


def test_pack_examples_from_pages():
    # 8 x 3-bit indices fill exactly 3 bytes (turboquant_pro, "How It Works").
    idx = np.array([[1, 2, 3, 4, 5, 6, 7, 0]])
    p = O.pack_bits(idx, 3)
    assert p.shape == (1, 3)
    stream = sum(int(v) << (3 * j) for j, v in enumerate(idx[0]))
    assert int.from_bytes(bytes(p[0]), "little") == stream
    # 4-bit: byte m = idx[2m] | idx[2m+1] << 4; 8-bit: one byte per index.
    idx4 = np.array([[3, 12, 15, 0]])
    assert O.pack_bits(idx4, 4).tolist() == [[3 | 12 << 4, 15]]
    assert O.pack_bits(np.array([[200, 7]]), 8).tolist() == [[200, 7]]


@pytest.mark.parametrize("d,bits", [(64, 8), (128, 4), (128, 3), (128, 2), (256, 4)])
def test_encode_is_nearest_centroid(d, bits):
    t = _table(d, bits)
    rng = np.random.default_rng(0)
    u = rng.standard_normal(20000) / math.sqrt(d)
    idx = O.encode(u, t.boundaries)
    c = t.centroids.astype(np.float64)
    brute = np.argmin(np.abs(u[:, None] - c[None, :]), axis=1)
    # The fp32 boundaries sit within fp32 rounding of the exact midpoints.
    mid = 0.5 * (c[:-1] + c[1:])
    near = np.min(np.abs(u[:, None] - mid[None, :]), axis=1) < 1e-6
    assert np.all((idx == brute) | near)
    assert np.mean(idx == brute) > 0.999


def test_encode_ties_go_low():
    b = np.array([-0.5, 0.0, 0.5], dtype=np.float32)
    assert O.encode(np.array([-0.5, 0.0, 0.5, 0.25, -1.0, 1.0]), b).tolist() == [0, 1, 2, 2, 0, 3]


def test_zero_and_nonfinite_rows():
    d = 128
    t = _table(d, 4)
    s = O.rht_signs(d, 0)
    x = np.zeros((3, d))
    x[1, 5] = np.inf
    x[2, :] = 1.0
    idx, n, _, bad = O.quantize_rows(x, s, t)
    assert idx[0].tolist() == [7] * d and n[0] == 0.0
    assert bad.tolist() == [False, True, False]
    assert idx[1].tolist() == [0] * d
    assert np.isnan(n[1]) and n[1].view(np.uint32) == 0x7FC00000
    np.testing.assert_array_equal(O.dequantize_rows(idx[0], n[0], t, s), np.zeros(d))
    assert n[2] == np.float32(math.sqrt(d))


def test_quantize_rows_matches_explicit_rotation():
    d = 64
    t = _table(d, 8)
    s = O.rht_signs(d, 11)
    rng = np.random.default_rng(3)
    x = rng.standard_normal((40, d)) * 3
    idx, n, u, _ = O.quantize_rows(x, s, t)
    r = O.rht_matrix(d, s)
    u_ref = (x @ r.T) / np.linalg.norm(x, axis=1, keepdims=True)
    np.testing.assert_allclose(u, u_ref, atol=1e-14)
    np.testing.assert_array_equal(n, np.linalg.norm(x, axis=1).astype(np.float32))
    xh = O.dequantize_rows(idx, n, t, s)
    cos = np.sum(x * xh, 1) / np.linalg.norm(x, axis=1) / np.linalg.norm(xh, axis=1)
    assert np.all(cos > 0.999)


def test_quality_sanity_against_printed_cosines(golden):
    d = 256
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2000, d))
    s = O.rht_signs(d, 0)
    for bits, printed, tol in golden("quality_gaussian_kv.txt"):
        t = _table(d, int(bits))
        idx, n, _, _ = O.quantize_rows(x, s, t)
        xh = O.dequantize_rows(idx, n, t, s)
        cos = np.mean(np.sum(x * xh, 1) / np.linalg.norm(x, axis=1) / np.linalg.norm(xh, axis=1))
        assert abs(cos - float(printed)) <= float(tol), (bits, cos)


def test_quantize_append_slot_placement():
    d, h_kv, bs, nblk = 64, 2, 16, 4
    kt, vt = _table(d, 4), _table(d, 2)
    kb, vb = O.region_bytes(d, 4), O.region_bytes(d, 2)
    stride = kb + vb + 8                     # padded slot
    pages = np.full((nblk, bs, h_kv, stride), 0xA5, dtype=np.uint8)
    rng = np.random.default_rng(5)
    k = rng.standard_normal((5, h_kv, d))
    v = rng.standard_normal((5, h_kv, d))
    slots = np.array([17, -1, 0, 63, 40])
    out = O.quantize_append(pages, slots, k, v, kt, vt, sign_seed=2)
    s = O.rht_signs(d, 2)
    written = np.zeros((nblk, bs), dtype=bool)
    for tok, slot in enumerate(slots):
        if slot < 0:
            continue
        blk, row = slot // bs, slot % bs
        written[blk, row] = True
        for h in range(h_kv):
            ki, kn, _, _ = O.quantize_rows(k[tok, h], s, kt)
            vi, vn, _, _ = O.quantize_rows(v[tok, h], s, vt)
            region = out[blk, row, h]
            assert bytes(region[:kb - 4]) == bytes(O.pack_bits(ki, 4))
            assert np.frombuffer(bytes(region[kb - 4:kb]), "<f4")[0] == kn
            assert bytes(region[kb:kb + vb - 4]) == bytes(O.pack_bits(vi, 2))
            assert np.frombuffer(bytes(region[kb + vb - 4:kb + vb]), "<f4")[0] == vn
            assert np.all(region[kb + vb:] == 0xA5)   # padding untouched
    assert np.all(out[~written] == 0xA5)


def _region_by_hand(idx, norm32, bits):
    """Region bytes laid out by hand from the page diagram (TorbuQuant, "TQ4 page
    tensor": packed indices, then the fp32 norm): code j occupies stream bits
    [j*bits, (j+1)*bits), stream bit p is bit p % 8 of byte p // 8, and the norm
    follows as four little-endian bytes (struct, not numpy)."""
    nbytes = (len(idx) * bits + 7) // 8
    out = bytearray(nbytes)
    for j, code in enumerate(idx):
        for k in range(bits):
            if (int(code) >> k) & 1:
                p = j * bits + k
                out[p // 8] |= 1 << (p % 8)
    return bytes(out) + struct.pack("<f", float(norm32))


@pytest.mark.parametrize("bits", range(1, 9))
@pytest.mark.parametrize("d", [64, 128, 256])
def test_decode_region_reads_hand_built_regions(bits, d):
    rng = np.random.default_rng(100 * d + bits)
    for _ in range(3):
        idx = rng.integers(0, 1 << bits, size=d)
        # norms with four distinct bytes, so a shifted or reversed read shows
        norm = np.float32(rng.uniform(0.5, 3000.0))
        raw = _region_by_hand(idx, norm, bits)
        assert len(raw) == O.region_bytes(d, bits)
        got_idx, got_n = O.decode_region(np.frombuffer(raw, dtype=np.uint8), d, bits)
        np.testing.assert_array_equal(got_idx, idx)
        assert got_n.dtype == np.float32 and got_n == norm


@pytest.mark.parametrize("d,kbits,vbits,pad", [(128, 4, 4, 0), (128, 3, 2, 8), (64, 8, 1, 16),
                                               (256, 5, 7, 24)])
def test_decode_region_splits_a_padded_kv_slot(d, kbits, vbits, pad):
    # A whole slot: [K codes | K norm][V codes | V norm][padding], each region read
    # back from its own byte range of the slot.
    rng = np.random.default_rng(d + kbits + vbits + pad)
    ki = rng.integers(0, 1 << kbits, size=(5, d))
    vi = rng.integers(0, 1 << vbits, size=(5, d))
    kn = rng.uniform(0.1, 50.0, size=5).astype(np.float32)
    vn = rng.uniform(0.1, 50.0, size=5).astype(np.float32)
    slots = np.array([np.frombuffer(_region_by_hand(ki[r], kn[r], kbits)
                                    + _region_by_hand(vi[r], vn[r], vbits)
                                    + b"\xa5" * pad, dtype=np.uint8) for r in range(5)])
    kb, vb = O.region_bytes(d, kbits), O.region_bytes(d, vbits)
    assert slots.shape == (5, kb + vb + pad)
    gi, gn = O.decode_region(slots[:, :kb], d, kbits)
    np.testing.assert_array_equal(gi, ki)
    np.testing.assert_array_equal(gn, kn)
    gi, gn = O.decode_region(slots[:, kb:kb + vb], d, vbits)
    np.testing.assert_array_equal(gi, vi)
    np.testing.assert_array_equal(gn, vn)


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_encode_region_matches_hand_layout_and_round_trips(bits):
    d = 128
    rng = np.random.default_rng(bits)
    idx = rng.integers(0, 1 << bits, size=(4, d))
    norm = rng.uniform(0.1, 9.0, size=4).astype(np.float32)
    reg = O.encode_region(idx, norm, bits)
    for r in range(4):
        assert bytes(reg[r]) == _region_by_hand(idx[r], norm[r], bits)
    gi, gn = O.decode_region(reg, d, bits)
    np.testing.assert_array_equal(gi, idx)
    np.testing.assert_array_equal(gn, norm)
