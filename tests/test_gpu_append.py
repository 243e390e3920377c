"""GPU parity of tq_quantize_append against the CPU oracle."""
import numpy as np
import pytest
import torch

from oracle import tq_oracle as O
from kv_cache_vector_append_b200 import workloads as W
from tests.gpu_helpers import gpu_append, oracle_table, require_gpu, to_np_f64

pytestmark = pytest.mark.gpu


def _tq():
    require_gpu()
    import kv_cache_vector_append_b200 as tq
    return tq


def _mini(d, kb, vb, dtype="bfloat16", h_kv=3, batch=3, seq=37, seed=7, **kw):
    return W.WorkloadSpec(f"mini-d{d}", d, h_kv, h_kv, batch, kb, vb, dtype, seq_len=seq,
                          n_outliers=2, outlier_factor=20.0, seed=seed, **kw)


def _regions(pages_np, wl, tokens, kind):
    """[n_tokens, H_kv, region] bytes of K (kind 0) or V (kind 1) for the given tokens."""
    d = wl.spec.head_dim
    kb = O.region_bytes(d, wl.spec.k_bits)
    vb = O.region_bytes(d, wl.spec.v_bits)
    slots = wl.slot_mapping[tokens]
    rows = pages_np[slots // 16, slots % 16]            # [n, H_kv, stride]
    return rows[..., :kb] if kind == 0 else rows[..., kb:kb + vb]


def _bit_exact_case(tq, wl, tokens=None, kind="beta", slot_stride=None, fill=0):
    """Packed bytes equal the oracle's packing of the GPU's own fp32 unit coords."""
    pages, cb = gpu_append(tq, wl, tokens, kind=kind, slot_stride=slot_stride, fill=fill)
    pages_np = pages.cpu().numpy()
    toks = np.arange(wl.k.shape[0]) if tokens is None else np.asarray(tokens)
    d = wl.spec.head_dim
    for which, (src, bits) in enumerate(((wl.k, wl.spec.k_bits), (wl.v, wl.spec.v_bits))):
        x = src[torch.from_numpy(toks)].reshape(-1, d).cuda()
        u = torch.empty(x.shape, dtype=torch.float32, device="cuda")
        n = torch.empty(x.shape[0], dtype=torch.float32, device="cuda")
        tq.rotate_unit(u, n, x, wl.spec.sign_seed)
        u_np = u.cpu().numpy().astype(np.float64)
        n_np = n.cpu().numpy()
        table = oracle_table(d, bits, kind)
        idx = O.encode(u_np, table.boundaries)
        expect = O.encode_region(idx, n_np, bits).reshape(len(toks), wl.spec.num_kv_heads, -1)
        got = _regions(pages_np, wl, toks, which)
        assert got.shape == expect.shape
        mism = np.nonzero(np.any(got != expect, axis=-1))
        assert mism[0].size == 0, f"region {which}: {mism[0].size} rows differ, first {mism[0][:5]}"
    return pages_np


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_bit_exact_all_bits(d, bits):
    tq = _tq()
    vb = 9 - bits
    _bit_exact_case(tq, W.generate(_mini(d, bits, vb, seed=bits)))


@pytest.mark.parametrize("dtype", ["float32", "bfloat16"])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_bit_exact_dtypes(d, dtype):
    tq = _tq()
    _bit_exact_case(tq, W.generate(_mini(d, 4, 2, dtype=dtype, batch=5, seq=53)))


def test_bit_exact_fp16_input():
    tq = _tq()
    wl = W.generate(_mini(128, 4, 4, dtype="float32", batch=2, seq=40))
    wl.k = wl.k.to(torch.float16)
    wl.v = wl.v.to(torch.float16)
    _bit_exact_case(tq, wl)


# Tiles of 2048 / D consecutive (token, head) pairs are staged by tensor copies and
# stored by one bulk copy per token when h_kv divides the tile (or the tile divides
# h_kv) and the pool's slots are packed with 16-byte alignment; h_kv = 3 above takes
# the cp.async staging and the per-word stores.  seq lengths leave ragged last tiles.
@pytest.mark.parametrize("d,h_kv,dtype,kb,vb", [
    (64, 8, "bfloat16", 4, 4), (128, 8, "bfloat16", 4, 4), (256, 8, "bfloat16", 3, 2),
    (128, 32, "bfloat16", 4, 2), (128, 2, "bfloat16", 8, 1), (128, 1, "bfloat16", 4, 4),
    (64, 16, "bfloat16", 2, 2), (256, 16, "bfloat16", 4, 4), (128, 8, "float32", 4, 4)])
def test_bit_exact_tile_copy_modes(d, h_kv, dtype, kb, vb):
    tq = _tq()
    _bit_exact_case(tq, W.generate(_mini(d, kb, vb, dtype=dtype, h_kv=h_kv, batch=3, seq=41,
                                         seed=h_kv + d)))


def test_bit_exact_fp16_tile_copy():
    tq = _tq()
    wl = W.generate(_mini(128, 4, 4, dtype="float32", h_kv=8, batch=2, seq=33))
    wl.k = wl.k.to(torch.float16)
    wl.v = wl.v.to(torch.float16)
    _bit_exact_case(tq, wl)


def test_strided_inputs_match_contiguous():
    """K and V as views into wider buffers (head stride 2D, token stride 2 h_kv D) give
    the same pages as contiguous inputs."""
    tq = _tq()
    wl = W.generate(_mini(128, 4, 2, h_kv=8, batch=2, seq=45))
    ref, cb = gpu_append(tq, wl)
    t, h, d = wl.k.shape
    wide_k = torch.zeros(t, h, 2 * d, dtype=wl.k.dtype)
    wide_v = torch.zeros(t, h, 2 * d, dtype=wl.v.dtype)
    wide_k[..., :d] = wl.k
    wide_v[..., d:] = wl.v
    k = wide_k.cuda()[..., :d]
    v = wide_v.cuda()[..., d:]
    pages = W.empty_pages(wl, device="cuda")
    sm = torch.from_numpy(wl.slot_mapping.astype(np.int64)).cuda()
    tq.quantize_append(pages, sm, k, v, cb, wl.spec.sign_seed)
    torch.cuda.synchronize()
    assert torch.equal(pages, ref)


def test_skipped_tokens_with_token_stores():
    """Tokens with slot -1 leave their slots untouched when slots are stored per token."""
    tq = _tq()
    wl = W.generate(_mini(128, 4, 4, h_kv=8, batch=2, seq=40))
    sm = wl.slot_mapping.copy()
    sm[1::3] = -1
    pages, _ = gpu_append(tq, wl, fill=0xA5, slot_mapping=sm)
    p = pages.cpu().numpy()
    written = np.zeros(p.shape[:2], dtype=bool)
    ok = sm >= 0
    written[sm[ok] // 16, sm[ok] % 16] = True
    assert np.all(p[~written] == 0xA5)
    full, _ = gpu_append(tq, wl)
    f = full.cpu().numpy()
    assert np.array_equal(p[written], f[written])


def _end_to_end(tq, wl, tokens=None, max_rows=None, kind="beta"):
    """Oracle fp64 vs GPU: >= 99.99% identical codes, every mismatch within 1e-5 of a
    boundary; norms within 1e-6 relative."""
    pages, _ = gpu_append(tq, wl, tokens, kind=kind)
    pages_np = pages.cpu().numpy()
    toks = np.arange(wl.k.shape[0]) if tokens is None else np.asarray(tokens)
    d = wl.spec.head_dim
    signs = O.rht_signs(d, wl.spec.sign_seed)
    total = mism = 0
    for which, (src, bits) in enumerate(((wl.k, wl.spec.k_bits), (wl.v, wl.spec.v_bits))):
        table = oracle_table(d, bits, kind)
        x = to_np_f64(src[torch.from_numpy(toks)])
        ref_idx, ref_n, ref_u, _ = O.quantize_rows(x, signs, table)
        got_idx, got_n = O.decode_region(_regions(pages_np, wl, toks, which), d, bits)
        np.testing.assert_allclose(got_n, ref_n, rtol=1e-6, atol=0)
        bad = got_idx != ref_idx
        total += bad.size
        mism += int(bad.sum())
        if bad.any():
            b = table.boundaries.astype(np.float64)
            dist = np.min(np.abs(ref_u[bad][:, None] - b[None, :]), axis=1)
            assert np.all(dist < 1e-5), f"mismatch far from a boundary: {dist.max()}"
    assert mism <= 1e-4 * total, f"{mism} of {total} codes differ"


@pytest.mark.parametrize("d,kb,vb", [(64, 8, 8), (128, 4, 4), (128, 4, 2), (128, 3, 2),
                                     (256, 4, 4), (256, 8, 2)])
def test_end_to_end_codes_and_norms(d, kb, vb):
    tq = _tq()
    _end_to_end(tq, W.generate(_mini(d, kb, vb, h_kv=4, batch=4, seq=301, seed=d + kb)))


def test_config0_end_to_end_and_bit_exact():
    tq = _tq()
    wl = W.generate(W.CONFIGS[0])
    _end_to_end(tq, wl)
    _bit_exact_case(tq, wl)


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_full_size_configs_sampled(cfg):
    # The whole configuration is appended in the launch shape the bench uses;
    # a seeded sample of tokens is checked against the oracle.
    tq = _tq()
    wl = W.generate(W.CONFIGS[cfg])
    pages, _ = gpu_append(tq, wl)
    pages_np = pages.cpu().numpy()
    rng = np.random.default_rng(cfg)
    toks = np.sort(rng.choice(wl.k.shape[0], size=min(3000, wl.k.shape[0]), replace=False))
    d = wl.spec.head_dim
    signs = O.rht_signs(d, wl.spec.sign_seed)
    mism = total = 0
    for kind, (src, bits) in enumerate(((wl.k, wl.spec.k_bits), (wl.v, wl.spec.v_bits))):
        table = oracle_table(d, bits)
        ref_idx, ref_n, ref_u, _ = O.quantize_rows(to_np_f64(src[torch.from_numpy(toks)]), signs,
                                                   table)
        got_idx, got_n = O.decode_region(_regions(pages_np, wl, toks, kind), d, bits)
        np.testing.assert_allclose(got_n, ref_n, rtol=1e-6, atol=0)
        bad = got_idx != ref_idx
        mism += int(bad.sum())
        total += bad.size
        if bad.any():
            b = table.boundaries.astype(np.float64)
            assert np.all(np.min(np.abs(ref_u[bad][:, None] - b[None, :]), axis=1) < 1e-5)
    assert mism <= 1e-4 * total


# A padded slot stride stores the slots one by one: with a stride that is a multiple of
# 16 bytes (pads 8 and 24 here), each slot's 16-byte body by a bulk copy and its tail by
# words; otherwise (pad 16) word by word.  Both write the oracle's bytes and leave the
# padding alone.
@pytest.mark.parametrize("pad", [8, 16, 24])
@pytest.mark.parametrize("d,kb,vb", [(128, 4, 2), (128, 4, 4), (64, 3, 3)])
def test_bit_exact_padded_slot_stride(d, kb, vb, pad):
    tq = _tq()
    wl = W.generate(_mini(d, kb, vb, h_kv=4, batch=3, seq=45, seed=pad + kb))
    pages_np = _bit_exact_case(tq, wl, slot_stride=wl.slot_bytes + pad, fill=0xA5)
    assert np.all(pages_np[..., wl.slot_bytes:] == 0xA5)


def test_padding_and_unmapped_slots_untouched():
    tq = _tq()
    wl = W.generate(_mini(128, 4, 2, batch=2, seq=40))
    stride = wl.slot_bytes + 24
    sm = wl.slot_mapping.copy()
    sm[::5] = -1                                    # skipped tokens
    pages, _ = gpu_append(tq, wl, pages=None, slot_stride=stride, fill=0xA5, slot_mapping=sm)
    p = pages.cpu().numpy()
    assert np.all(p[..., wl.slot_bytes:] == 0xA5)
    written = np.zeros(p.shape[:2], dtype=bool)
    ok = sm >= 0
    written[sm[ok] // 16, sm[ok] % 16] = True
    assert np.all(p[~written] == 0xA5)
    # written slots hold the oracle's regions (bit-exact path on the kept tokens)
    assert not np.all(p[written][..., :wl.slot_bytes] == 0xA5)


def test_zero_nonfinite_and_out_of_range_rows():
    tq = _tq()
    spec = _mini(128, 4, 4, dtype="float32", h_kv=2, batch=1, seq=20)
    wl = W.generate(spec)
    wl.k[3] = 0.0                       # zero row (both heads)
    wl.v[5, 1, 7] = float("nan")
    wl.k[6, 0, 0] = float("inf")
    sm = wl.slot_mapping.copy()
    sm[10] = wl.num_blocks * 16 + 5     # out of range -> skipped, error bit
    tq.get_device_error()               # clear
    pages, _ = gpu_append(tq, wl, fill=0x5A, slot_mapping=sm)
    err = tq.get_device_error()
    assert err & tq.DEVERR_SLOT_RANGE and err & tq.DEVERR_NONFINITE
    p = pages.cpu().numpy()
    kb = O.region_bytes(128, 4)
    # zero row: norm 0, codes idx(0) = 7
    zr = _regions(p, wl, np.array([3]), 0)[0]
    idx, n = O.decode_region(zr, 128, 4)
    assert np.all(n == 0) and np.all(idx == 7)
    # non-finite rows: codes 0, quiet-NaN norm
    vr = _regions(p, wl, np.array([5]), 1)[0, 1]
    kr = _regions(p, wl, np.array([6]), 0)[0, 0]
    for r, bits in ((vr, 4), (kr, 4)):
        i, n = O.decode_region(r, 128, bits)
        assert np.all(i == 0) and n.view(np.uint32) == 0x7FC00000
    # the other head of token 6 is a normal row
    i, n = O.decode_region(_regions(p, wl, np.array([6]), 0)[0, 1], 128, 4)
    assert np.isfinite(n) and n > 0
    assert tq.get_device_error() == 0   # read clears


def _scale_tokens(wl, scales):
    """Multiply token t's K and V rows by scales[t % len(scales)] (in fp32, then stored
    in the workload's dtype), so that every warp tile mixes row magnitudes."""
    f = torch.tensor([scales[t % len(scales)] for t in range(wl.k.shape[0])],
                     dtype=torch.float64)[:, None, None]
    wl.k = (wl.k.double() * f).to(wl.k.dtype)
    wl.v = (wl.v.double() * f).to(wl.v.dtype)
    return wl


# The method is scale-free (u = y / n), so rows far from unit scale must encode like
# unit-scale rows and keep their norm to 1e-6 relative: squares of 1e30 overflow fp32
# and squares of 1e-20 are subnormal, so the kernel rescales such rows exactly.
@pytest.mark.parametrize("dtype,scales", [
    ("float32", [1.0, 1e-30, 1e30, 1e-20, 1e18, 1.0, 1e-37, 3e36]),
    ("bfloat16", [1.0, 1e-35, 1e35, 1e-20, 1e18]),
])
def test_extreme_row_magnitudes(dtype, scales):
    tq = _tq()
    for d in (64, 128, 256):
        wl = _scale_tokens(W.generate(_mini(d, 4, 3, dtype=dtype, h_kv=8, batch=2, seq=40,
                                             seed=d)), scales)
        _bit_exact_case(tq, wl)
        _end_to_end(tq, wl)


def test_norm_beyond_fp32_range_stores_inf():
    # bf16 rows of 2e38 everywhere: ||x|| = 2e38 sqrt(D) exceeds fp32; the codes are
    # still those of the unit row and the stored norm is +inf (the oracle's fp32 norm).
    tq = _tq()
    wl = W.generate(_mini(128, 4, 4, dtype="bfloat16", h_kv=2, batch=1, seq=8, seed=3))
    wl.k[2] = 2e38
    wl.v[5, 1] = -2e38
    tq.get_device_error()
    _end_to_end(tq, wl)
    pages, _ = gpu_append(tq, wl)
    p = pages.cpu().numpy()
    _, n = O.decode_region(_regions(p, wl, np.array([2]), 0)[0], 128, 4)
    assert np.all(np.isposinf(n))
    assert tq.get_device_error() == 0    # a finite row is not an error


@pytest.mark.parametrize("d,kb,vb", [(128, 4, 2), (64, 3, 8), (256, 2, 4)])
def test_gaussian_codebooks(d, kb, vb):
    # The Gaussian-approximation tables (N(0, 1/D)) go through the same kernels.
    tq = _tq()
    wl = W.generate(_mini(d, kb, vb, h_kv=8, batch=2, seq=45, seed=d + 5))
    _bit_exact_case(tq, wl, kind="gauss")
    _end_to_end(tq, wl, kind="gauss")
