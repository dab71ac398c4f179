"""Pins for the oracle's Philox4x32-10 and uniform vocabulary draws."""
import os

import numpy as np
import pytest
from scipy import stats

from oracle.philox import philox4x32_10, uniform_ids

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _kat():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append([int(f, 16) for f in line.split()])
    return rows


@pytest.mark.parametrize("row", _kat())
def test_known_answer_vectors(row):
    c0, c1, c2, c3, k0, k1 = row[:6]
    out = philox4x32_10(c0, c1, c2, c3, k0, k1)
    assert [int(o) for o in out] == row[6:]


def test_vectorised_matches_scalar():
    rng = np.random.default_rng(1)
    c = rng.integers(0, 2**32, size=(4, 64), dtype=np.uint64)
    k = rng.integers(0, 2**32, size=2, dtype=np.uint64)
    vec = philox4x32_10(c[0], c[1], c[2], c[3], int(k[0]), int(k[1]))
    for j in range(64):
        sc = philox4x32_10(int(c[0, j]), int(c[1, j]), int(c[2, j]), int(c[3, j]), int(k[0]), int(k[1]))
        assert [int(v[j]) for v in vec] == [int(s) for s in sc]


def test_id_is_top_bits_for_power_of_two_vocab():
    # floor(r0 * 2^k / 2^32) is r0 >> (32 - k)
    pos = np.arange(4096)
    seed = 0x1234_5678_9ABC_DEF0
    r0 = philox4x32_10(pos, 7, 3, 1, seed & 0xFFFFFFFF, seed >> 32)[0]
    for bits in (12, 18):
        ids = uniform_ids(seed, 3, 7, pos, 1, 1 << bits)
        assert np.array_equal(ids, (r0 >> np.uint64(32 - bits)).astype(np.int64))


def test_ids_uniform_chi_square():
    n, vocab = 1 << 20, 1024
    ids = uniform_ids(0, 0, 0, np.arange(n), 0, vocab)
    assert ids.min() >= 0 and ids.max() < vocab
    counts = np.bincount(ids, minlength=vocab)
    chi2 = ((counts - n / vocab) ** 2 / (n / vocab)).sum()
    p = stats.chi2.sf(chi2, vocab - 1)
    assert 1e-4 < p < 1 - 1e-4


def test_counter_fields_are_distinct_streams():
    # changing any one counter field or the seed changes the draw stream
    pos = np.arange(256)
    base = uniform_ids(5, 1, 2, pos, 1, 1 << 18)
    for other in (uniform_ids(6, 1, 2, pos, 1, 1 << 18), uniform_ids(5, 2, 2, pos, 1, 1 << 18),
                  uniform_ids(5, 1, 3, pos, 1, 1 << 18), uniform_ids(5, 1, 2, pos, 0, 1 << 18),
                  uniform_ids(5 + (1 << 32), 1, 2, pos, 1, 1 << 18)):
        assert (base != other).mean() > 0.99
