"""Host-only checks of the decode kernel's shared-memory plan (tq_decode_plan_probe).

The decode kernel places, inside its dynamic shared memory: the code-pair lookup
tables at a shared-window address that is a multiple of 65536, a ring of stages (one
staged page block per warp group) below and above the tables, and a misc area at the
bottom or the top.  These tests check that every planned region lies inside the budget,
that no two regions overlap, and that copy destinations keep the 16-byte alignment the
bulk and tensor copies need, across the benchmark geometries and edge cases, for a
B200-like device (148 SMs, 227 KiB per CTA) and several window bases.
"""
import pytest

from kv_cache_vector_append_b200 import _binding as B

SMS, BUDGET = 148, 227 * 1024


def _probe(batch, h_q, h_kv, d, kb, vb, stride, max_blocks, base):
    r = B.decode_plan_probe(batch, h_q, h_kv, d, kb, vb, stride, max_blocks, SMS, BUDGET, base)
    return (B.OK, r) if isinstance(r, dict) else (r, None)


def _slot(d, kb, vb):
    return (d * kb + 7) // 8 + 4 + (d * vb + 7) // 8 + 4


GEOMS = [  # batch, h_q, h_kv, D, k_bits, v_bits, slot stride, max_blocks
    (8, 14, 2, 64, 8, 8, None, 256),
    (32, 32, 8, 128, 4, 4, None, 512),
    (64, 28, 4, 128, 4, 2, None, 2048),
    (1, 32, 8, 128, 3, 2, None, 8192),
    (1, 1, 1, 128, 4, 4, None, 16),
    (4, 16, 1, 128, 2, 2, None, 64),         # G = 16
    (2, 64, 8, 256, 4, 4, None, 32),         # D = 256
    (3, 24, 4, 256, 8, 8, None, 40),
    (2, 16, 8, 128, 8, 8, None, 40),
    (5, 12, 4, 64, 1, 1, None, 7),
    (2, 32, 8, 128, 4, 4, 160, 100),         # padded slots
    (1024, 32, 8, 128, 4, 4, None, 4),       # many short sequences
]


@pytest.mark.parametrize("base", [0, 16, 1024])
@pytest.mark.parametrize("g", GEOMS)
def test_plan_regions_fit_and_do_not_overlap(g, base):
    batch, h_q, h_kv, d, kb, vb, stride, max_blocks = g
    stride = stride or _slot(d, kb, vb)
    s, p = _probe(batch, h_q, h_kv, d, kb, vb, stride, max_blocks, base)
    assert s == B.OK, s
    assert p["lut_win"] % 65536 == 0 and p["lut_win"] == base + p["lut_off"]
    assert 0 <= p["smem"] <= BUDGET
    assert p["wph"] * h_kv <= p["warps"]
    assert (2 if p["wph"] == 1 else 4) <= p["nst"] <= 8
    assert 0 <= p["n_low"] <= p["nst"]
    # rows: whole slots of every KV head; a 2-D box also pads them to 20 (mod 32) words
    row_bytes = h_kv * stride
    if p["copy_mode"]:
        assert p["row_pitch"] >= row_bytes and (p["row_pitch"] // 4) % 32 == 20
        assert p["row_pitch"] // 8 <= 256 and row_bytes % 16 == 0
    else:
        assert p["row_pitch"] == row_bytes
    assert p["stage_bytes"] == p["wph"] * 16 * p["row_pitch"]
    # regions [start, end)
    lut = (p["lut_off"], p["lut_off"] + p["lut_bytes"])
    lo = (p["stage_lo_off"], p["stage_lo_off"] + p["n_low"] * p["stage_bytes"])
    hi = (p["stage_hi_off"], p["stage_hi_off"] + (p["nst"] - p["n_low"]) * p["stage_bytes"])
    assert lo[1] == lut[0] if p["n_low"] else True          # low stages end at the tables
    assert hi[0] == lut[1]                                   # high stages start after them
    misc_top = p["misc_off"] > 0
    if misc_top:
        misc = (p["misc_off"], p["smem"])
        assert misc[0] >= hi[1] and misc[0] % 16 == 0
    else:
        misc = (0, lo[0] if p["n_low"] else lut[0])          # misc fills what is below
        assert misc[1] > 0
    regions = [r for r in (lut, lo, hi, misc) if r[1] > r[0]]
    for r in regions:
        assert 0 <= r[0] < r[1] <= p["smem"]
    regions.sort()
    for a, b in zip(regions, regions[1:]):
        assert a[1] <= b[0], (a, b)
    # copy destinations: 16-byte aligned shared-window addresses
    for k in range(p["n_low"]):
        assert (base + lo[0] + k * p["stage_bytes"]) % 16 == 0
    for k in range(p["nst"] - p["n_low"]):
        assert (base + hi[0] + k * p["stage_bytes"]) % 16 == 0


def test_plan_rejects_impossible_geometries():
    assert _probe(2, 64, 32, 128, 4, 4, 136, 8, 0)[0] == B.ERR_UNSUPPORTED   # 32 KV heads
    assert _probe(2, 32, 16, 256, 4, 4, 264, 8, 0)[0] == B.ERR_UNSUPPORTED  # > 8 at D=256
    # 8-bit tables (64 KiB, on a 64 KiB boundary) leave no room for two staged blocks
    assert _probe(2, 16, 16, 128, 8, 8, 264, 8, 0)[0] == B.ERR_UNSUPPORTED
    assert _probe(2, 16, 8, 256, 8, 8, 520, 8, 0)[0] == B.ERR_UNSUPPORTED
    assert _probe(2, 32, 8, 128, 4, 4, 136, 8, 0)[0] == B.OK
    assert _probe(0, 32, 8, 128, 4, 4, 136, 8, 0)[0] == B.ERR_INVALID_ARG
    assert _probe(2, 30, 8, 128, 4, 4, 136, 8, 0)[0] == B.ERR_INVALID_ARG    # 30 % 8
