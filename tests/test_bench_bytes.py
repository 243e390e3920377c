"""The algorithmic bytes behind the bench's roofline: per (token, KV head) the append
reads two input rows and writes one slot, the decode reads one slot; both also count
their index arrays and the query/output rows.  The slot sizes come from the oracle's
page layout (plain and QJL), and the totals are counted here row by row, not by the
bench's closed forms."""

import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from oracle import tq_oracle as O  # noqa: E402
from kv_cache_vector_append_b200 import workloads as W  # noqa: E402


def _slot(spec, qjl=False):
    return (O.k_region_bytes(spec.head_dim, spec.k_bits, qjl)
            + O.region_bytes(spec.head_dim, spec.v_bits))


def _counted_append(spec, n_tokens, slot):
    es = np.dtype(np.float32).itemsize if spec.dtype == "float32" else 2
    total = 0
    for _ in range(n_tokens):
        total += 8                                        # its slot_mapping entry
        for _ in range(spec.num_kv_heads):
            total += 2 * spec.head_dim * es + slot        # K and V rows in, one slot out
    return total


def _counted_decode(spec, seq_lens, slot):
    es = np.dtype(np.float32).itemsize if spec.dtype == "float32" else 2
    packed = table = 0
    for n in seq_lens:
        packed += int(n) * spec.num_kv_heads * slot
        table += 4 * -(-int(n) // 16)                     # one i32 per 16-token block
    rows = 2 * len(seq_lens) * spec.num_q_heads * spec.head_dim * es
    return packed + table + rows, packed


@pytest.mark.parametrize("cfg", [0, 2, 3, 4])
def test_plain_slot_bytes(cfg):
    spec = W.CONFIGS[cfg]
    wl = W.generate(spec.scaled(batch=2) if cfg in (2, 3) else spec)
    n = len(wl.step_tokens)
    assert bench.append_bytes(wl.spec, n) == _counted_append(wl.spec, n, _slot(wl.spec))
    assert bench.decode_bytes(wl.spec, wl.seq_lens) == _counted_decode(
        wl.spec, wl.seq_lens, _slot(wl.spec))


def test_qjl_slot_bytes():
    spec = W.CONFIGS[2].scaled(batch=2)
    wl = W.generate(spec)
    sb = _slot(spec, qjl=True)
    assert sb == _slot(spec) + spec.head_dim // 8 + 4    # D sign bits and gamma
    n = len(wl.step_tokens)
    assert bench.append_bytes(spec, n, sb) == _counted_append(spec, n, sb)
    assert bench.decode_bytes(spec, wl.seq_lens, sb) == _counted_decode(spec, wl.seq_lens, sb)


def test_leg_summary_uses_the_given_slot():
    spec = W.CONFIGS[2].scaled(batch=2)
    wl = W.generate(spec)
    sb = _slot(spec, qjl=True)
    leg = bench.leg_summary(wl, 1.0, 1.0, 1000.0, sb=sb)
    assert leg["append"]["bytes"] == _counted_append(spec, len(wl.step_tokens), sb)
    assert leg["decode"]["bytes"] == _counted_decode(spec, wl.seq_lens, sb)[0]
    # 1 ms per leg: GB/s is bytes / 1e6
    assert leg["decode"]["gbs"] == pytest.approx(leg["decode"]["bytes"] / 1e6)
