"""Pins of the oracle's sign generator (SplitMix64) and sign vector."""
import numpy as np
import pandas as pd
import pytest

from oracle import tq_oracle as O


def test_splitmix64_published_outputs(golden):
    for seed, index, hexval in golden("splitmix64.txt"):
        z = O.splitmix64_outputs(int(seed), int(index) + 1)
        assert int(z[int(index)]) == int(hexval, 16)


@pytest.mark.parametrize("seed", [0, 1, 12345, 2**63 + 7, 2**64 - 1])
def test_splitmix64_matches_independent_finalizer(seed):
    # pandas.util.hash_array applies the SplitMix64 finalizer to uint64 input;
    # feed it the generator states seed + (j+1)*gamma.
    n = 300
    states = np.array([(seed + (j + 1) * O.SPLITMIX64_GAMMA) % 2**64 for j in range(n)],
                      dtype=np.uint64)
    ref = pd.util.hash_array(states)
    np.testing.assert_array_equal(O.splitmix64_outputs(seed, n), ref)


def test_sign_vector_values_and_balance():
    s = O.rht_signs(1 << 16, 0)
    assert set(np.unique(s)) == {-1.0, 1.0}
    frac = np.mean(s < 0)
    assert abs(frac - 0.5) < 4 * 0.5 / np.sqrt(s.size)
    # seeds give different vectors; the vector is a prefix-stable stream
    assert not np.array_equal(O.rht_signs(128, 0), O.rht_signs(128, 1))
    np.testing.assert_array_equal(O.rht_signs(64, 5), O.rht_signs(256, 5)[:64])


def test_sign_is_top_bit():
    z = O.splitmix64_outputs(3, 64)
    s = O.rht_signs(64, 3)
    for j in range(64):
        assert (s[j] < 0) == (int(z[j]) >= 2**63)
