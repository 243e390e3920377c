"""Planted mistakes in the oracle (on the CPU) must fail at least one pin.

Each case monkeypatches one oracle function with a plausible slip and runs the
pins that should catch it.
"""
import math

import numpy as np
import pytest

from oracle import tq_oracle as O
from tests.conftest import read_golden
from tests import test_oracle_attention as TA
from tests import test_oracle_codebook as TC
from tests import test_oracle_pack_encode as TP
from tests import test_oracle_rotation as TR
from tests import test_oracle_signs as TS


def _fails(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_mutation_fwht_butterfly_sign(monkeypatch):
    orig = O.fwht

    def bad(x):
        return orig(x)[..., ::-1]
    monkeypatch.setattr(O, "fwht", bad)
    _fails(TR.test_fwht_equals_explicit_product, 8)


def test_mutation_signs_after_transform(monkeypatch):
    def bad(x, signs):
        return O.fwht(np.asarray(x, dtype=np.float64)) * signs / math.sqrt(x.shape[-1])
    monkeypatch.setattr(O, "rht_forward", bad)
    _fails(TR.test_rht_signs_applied_before_transform)


def test_mutation_sign_bit_choice(monkeypatch):
    def bad(dim, seed):
        z = O.splitmix64_outputs(seed, dim)
        return np.where((z & np.uint64(1)) == 1, -1.0, 1.0)
    monkeypatch.setattr(O, "rht_signs", bad)
    _fails(TS.test_sign_is_top_bit)


def test_mutation_density_exponent(monkeypatch):
    orig_init = O.BetaSphereDensity.__init__

    def bad_init(self, dim):
        orig_init(self, dim)
        self.a = (dim - 2) / 2.0
    monkeypatch.setattr(O.BetaSphereDensity, "__init__", bad_init)
    _fails(TC.test_beta_density_matches_library, 64)


def test_mutation_lloyd_boundary(monkeypatch):
    # centroid update over the wrong cell edges (shifted by one)
    orig = O.GaussianDensity.first_moment

    def bad(self, lo, hi):
        return orig(self, lo, hi) * 1.01
    monkeypatch.setattr(O.GaussianDensity, "first_moment", bad)
    _fails(TC.test_gaussian_distortions_match_max_1960, read_golden)


def test_mutation_pack_msb_first(monkeypatch):
    def bad(idx, bits):
        rev = np.zeros_like(np.asarray(idx))
        for k in range(bits):
            rev |= ((np.asarray(idx) >> k) & 1) << (bits - 1 - k)
        return orig(rev, bits)
    orig = O.pack_bits
    monkeypatch.setattr(O, "pack_bits", bad)
    _fails(TP.test_pack_examples_from_pages)


def test_mutation_encode_tie_high(monkeypatch):
    def bad(u, boundaries):
        b = np.asarray(boundaries, dtype=np.float64)
        u = np.asarray(u, dtype=np.float64)
        return np.sum(b[None, :] <= u.reshape(-1, 1), axis=1).reshape(u.shape)
    monkeypatch.setattr(O, "encode", bad)
    _fails(TP.test_encode_ties_go_low)


def test_mutation_gqa_interleaved(monkeypatch):
    orig = O.paged_decode

    def bad(q, pages, bt, sl, kt, vt, seed, scale):
        # query head h reads KV head h % H_kv instead of h // G
        h_kv = pages.shape[2]
        out = np.zeros(q.shape)
        for h in range(q.shape[1]):
            out[:, h] = orig(q[:, h:h + 1], pages[:, :, h % h_kv:h % h_kv + 1], bt, sl, kt, vt,
                             seed, scale)[:, 0]
        return out
    monkeypatch.setattr(O, "paged_decode", bad)
    _fails(TA.test_gqa_grouping_is_contiguous)


def test_mutation_dequant_without_inverse_rotation(monkeypatch):
    def bad(idx, norm32, table, signs):
        c = np.asarray(table.centroids, dtype=np.float64)[np.asarray(idx)]
        return np.asarray(norm32, dtype=np.float64)[..., None] * c
    monkeypatch.setattr(O, "dequantize_rows", bad)
    _fails(TA.test_decode_brute_force, 64, 4, 2, 8, 8)


def test_mutation_merge_missing_rescale(monkeypatch):
    def bad(parts):
        return sum(p[2] for p in parts) / sum(p[1] for p in parts)
    monkeypatch.setattr(O, "merge_partials", bad)
    _fails(TA.test_rotated_domain_and_split_merge_equal_plain)


def test_mutation_region_norm_offset(monkeypatch):
    # the norm read four bytes early (from the last packed bytes)
    def bad(region, dim, bits):
        region = np.asarray(region, dtype=np.uint8)
        nb = (dim * bits + 7) // 8
        idx = O.unpack_bits(region[..., :nb], dim, bits)
        norm = np.ascontiguousarray(region[..., nb - 4:nb]).view("<f4")[..., 0]
        return idx, norm.astype(np.float32)
    monkeypatch.setattr(O, "decode_region", bad)
    _fails(TP.test_decode_region_reads_hand_built_regions, 4, 128)


def test_mutation_region_norm_first(monkeypatch):
    # the layout misread as [fp32 norm | packed codes]
    def bad(region, dim, bits):
        region = np.asarray(region, dtype=np.uint8)
        nb = (dim * bits + 7) // 8
        idx = O.unpack_bits(region[..., 4:4 + nb], dim, bits)
        norm = np.ascontiguousarray(region[..., :4]).view("<f4")[..., 0]
        return idx, norm.astype(np.float32)
    monkeypatch.setattr(O, "decode_region", bad)
    _fails(TP.test_decode_region_splits_a_padded_kv_slot, 128, 3, 2, 8)


def test_mutation_region_big_endian_norm(monkeypatch):
    def bad(region, dim, bits):
        region = np.asarray(region, dtype=np.uint8)
        nb = (dim * bits + 7) // 8
        idx = O.unpack_bits(region[..., :nb], dim, bits)
        norm = np.ascontiguousarray(region[..., nb:nb + 4]).view(">f4")[..., 0]
        return idx, norm.astype(np.float32)
    monkeypatch.setattr(O, "decode_region", bad)
    _fails(TP.test_decode_region_reads_hand_built_regions, 2, 64)


def test_mutation_hot_window_separate_softmax(monkeypatch):
    # packed and hot tokens normalised separately, then averaged
    orig = O.paged_decode_hot

    def bad(q, pages, bt, sl, hk, hv, hl, kt, vt, seed, scale):
        a = orig(q, pages, bt, sl, hk, hv, np.zeros_like(hl), kt, vt, seed, scale)
        b = orig(q, pages, bt, np.zeros_like(sl), hk, hv, hl, kt, vt, seed, scale)
        return 0.5 * (a + b)
    monkeypatch.setattr(O, "paged_decode_hot", bad)
    _fails(TA.test_hot_window_joins_the_packed_softmax)


def test_mutation_haar_without_sign_fix(monkeypatch):
    # numpy's QR factor used as it comes: the signs of R's diagonal left in R
    def bad(dim, seed):
        return np.linalg.qr(np.random.default_rng(seed).standard_normal((dim, dim)))[0]
    monkeypatch.setattr(O, "haar_orthogonal", bad)
    _fails(TR.test_haar_matrix_is_orthogonal_and_the_positive_diagonal_qr, 16)


def test_mutation_qjl_constant(monkeypatch):
    # sqrt(2/pi) in place of sqrt(pi/2): the estimator is biased by 2/pi
    monkeypatch.setattr(O, "QJL_CONST", math.sqrt(2.0 / math.pi))
    from tests import test_oracle_qjl as TQ
    _fails(TQ.test_qjl_estimator_is_unbiased_over_sketch_signs)
