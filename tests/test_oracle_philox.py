"""Pins of the oracle's counter-based RNG (Philox4x32-10 and the uniform)."""
from pathlib import Path

import numpy as np
import pytest

import oracle

KAT = Path(__file__).parent / "golden" / "philox4x32_10_kat.txt"


def _kat_rows():
    rows = []
    for line in KAT.read_text().splitlines():
        if not line.strip() or line.startswith("#"):
            continue
        w = [int(t, 16) for t in line.split()]
        rows.append((w[0:4], w[4:6], w[6:10]))
    return rows


@pytest.mark.parametrize("ctr,key,out", _kat_rows())
def test_philox_known_answers(ctr, key, out):
    assert list(oracle.philox(ctr, key)) == out


@pytest.mark.parametrize("ctr,key,out", _kat_rows())
def test_uniform_counter_layout(ctr, key, out):
    # counter = (request, position, draw, cycle); key = seed low word, high word;
    # u = (word0 * 2^21 + word1 >> 11) * 2^-53.
    seed = (key[1] << 32) | key[0]
    u = oracle.uniform(seed, ctr[0], ctr[1], ctr[2], ctr[3])
    m = (out[0] << 21) | (out[1] >> 11)
    assert u == m * 2.0 ** -53
    assert 0.0 <= u < 1.0


def test_uniform_distinct_streams():
    us = {oracle.uniform(42, r, p, d, c) for r in range(4) for p in range(4) for d in range(4) for c in range(2)}
    assert len(us) == 4 * 4 * 4 * 2


def test_uniform_is_uniform():
    from scipy import stats
    u = np.array([oracle.uniform(7, r, 3, 1, 0) for r in range(20000)])
    assert stats.kstest(u, "uniform").pvalue > 1e-4


def test_first_request_offsets_the_request_counter():
    # a slice of the batch with first_request = 3 draws what the whole batch
    # draws for requests 3..5 (the counter's request word is global)
    rng = np.random.default_rng(11)
    x = rng.standard_normal((6 * 2, 40)).astype(np.float32)
    whole = oracle.filter_softmax(x, "f32", 1.0, 10, 0.9, rows_per_request=2, rng=(5, 1))
    part = oracle.filter_softmax(x[6:], "f32", 1.0, 10, 0.9, rows_per_request=2, rng=(5, 1, 3))
    assert np.array_equal(part["sample"], whole["sample"][6:])
    # without the offset the slice draws request 0..2's uniforms instead
    for r in range(3):
        for p in range(2):
            assert oracle.uniform(5, 3 + r, p, 0, 1) != oracle.uniform(5, r, p, 0, 1)
