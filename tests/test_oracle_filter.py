"""Pins of the oracle's filter (temperature, top-k, top-p, softmax) and sampler."""
import numpy as np
import pytest
from scipy import special

import oracle
from _defs import bf16_to_f32, chi2_pvalue, filtered_dist, top_p_margin
from speculative_decoding_verification_filter_b200.inputs import to_bf16_bits


def _dense(out, vocab):
    rows = out["ids"].shape[0]
    d = np.zeros((rows, vocab))
    for r in range(rows):
        c = out["count"][r]
        d[r, out["ids"][r, :c]] = out["probs"][r, :c]
    return d


def test_greedy_is_argmax_with_lowest_id_on_ties():
    rng = np.random.default_rng(1)
    x = rng.integers(-3, 4, size=(64, 37)).astype(np.float32)  # many ties
    for T, k in [(0.0, 50), (1.0, 1), (0.5, 1)]:
        out = oracle.filter_softmax(x, "f32", T, k, 0.9, cap=50)
        assert np.all(out["count"] == 1)
        assert np.array_equal(out["ids"][:, 0], np.argmax(x, axis=1))  # argmax: first maximum
        assert np.all(out["probs"][:, 0] == 1.0)


def test_full_softmax_when_nothing_is_cut():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((16, 40)) * 2).astype(np.float32)
    for T in (1.0, 0.7, 1.9):
        out = oracle.filter_softmax(x, "f32", T, 40, 1.0, dense=True)
        ref = special.softmax(x.astype(np.float64) / T, axis=1)
        assert np.all(out["count"] == 40)
        assert np.max(np.abs(out["dense"] - ref)) < 1e-7


def test_top_k_softmax_matches_library_top_k():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((32, 200)).astype(np.float32)
    x[:, 5] = x[:, 7]  # a tie that top-k must break by id
    for k in (1, 5, 50, 199):
        out = oracle.filter_softmax(x, "f32", 1.0, k, 1.0)
        for r in range(x.shape[0]):
            order = np.lexsort((np.arange(200), -x[r].astype(np.float64)))[:k]
            c = out["count"][r]
            assert c == k
            assert np.array_equal(out["ids"][r, :c], np.sort(order))
            ref = special.softmax(x[r, np.sort(order)].astype(np.float64))
            assert np.max(np.abs(out["probs"][r, :c] - ref)) < 1e-7


@pytest.mark.parametrize("T,k,p", [(1.0, 50, 0.95), (0.7, 50, 0.9), (1.3, 20, 0.5), (1.0, 100, 0.999),
                                   (1.0, 3, 0.2)])
def test_top_p_is_shortest_prefix_reaching_top_p(T, k, p):
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((200, 300)) * 1.5).astype(np.float32)
    out = oracle.filter_softmax(x, "f32", T, k, p, dense=True)
    checked = 0
    for r in range(x.shape[0]):
        if top_p_margin(x[r], T, k, p) < 1e-9:
            continue
        ref = filtered_dist(x[r], T, k, p)
        assert out["count"][r] == np.count_nonzero(ref)
        assert np.max(np.abs(out["dense"][r] - ref)) < 1e-7
        checked += 1
    assert checked > 190


def test_compact_output_invariants():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((100, 500)) * 3).astype(np.float32)
    out = oracle.filter_softmax(x, "f32", 1.0, 50, 0.95, cap=64, dense=True)
    for r in range(100):
        c = out["count"][r]
        assert 1 <= c <= 50
        ids, pr = out["ids"][r, :c], out["probs"][r, :c]
        assert np.all(np.diff(ids) > 0)  # ascending ids
        assert abs(pr.astype(np.float64).sum() - 1.0) < 1e-6
        # probabilities are monotone in the logit
        o = np.argsort(-x[r, ids], kind="stable")
        assert np.all(np.diff(pr[o]) <= 0)
        assert np.all(out["ids"][r, c:] == -1) and np.all(out["probs"][r, c:] == 0)
        assert np.array_equal(np.nonzero(out["dense"][r])[0], ids)


def test_bf16_rows_filter_as_their_decoded_values():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((20, 333)).astype(np.float32)
    bits = to_bf16_bits(x)
    a = oracle.filter_softmax(bits, "bf16", 1.0, 50, 0.95)
    b = oracle.filter_softmax(bf16_to_f32(bits), "f32", 1.0, 50, 0.95)
    for key in ("ids", "probs", "count"):
        assert np.array_equal(a[key], b[key])


def test_non_finite_rows_and_masked_tokens():
    x = np.zeros((5, 10), dtype=np.float32)
    x[0, 3] = np.nan
    x[1, 4] = np.inf
    x[2, :] = -np.inf
    x[3, :] = -np.inf
    x[3, 6] = 1.0
    x[3, 2] = 0.5  # two finite tokens, top_k 5
    x[4, :] = np.arange(10)
    x[4, 9] = -np.inf  # the would-be argmax is masked
    out = oracle.filter_softmax(x, "f32", 1.0, 5, 1.0, rng=(3, 0))
    assert list(out["flags"][:3]) == [oracle.FLAG_NONFINITE_ROW] * 3
    assert list(out["count"][:3]) == [0, 0, 0]
    assert list(out["sample"][:3]) == [-1, -1, -1]
    assert out["count"][3] == 2 and list(out["ids"][3, :2]) == [2, 6]
    assert out["flags"][3] == 0
    assert list(out["ids"][4, :5]) == [4, 5, 6, 7, 8]


def test_temperature_is_a_logit_scale():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((10, 64)).astype(np.float64)
    T = 0.5
    a = oracle.filter_softmax(x.astype(np.float32), "f32", T, 64, 1.0, dense=True)
    ref = special.softmax(x.astype(np.float32).astype(np.float64) / T, axis=1)
    assert np.max(np.abs(a["dense"] - ref)) < 1e-7


def test_k_at_least_vocab_is_clamped():
    x = np.linspace(-1, 1, 7, dtype=np.float32)[None, :]
    out = oracle.filter_softmax(x, "f32", 1.0, 1000, 1.0, cap=7)
    assert out["count"][0] == 7


def test_sampler_matches_filtered_distribution():
    rng = np.random.default_rng(8)
    base = (rng.standard_normal(12) * 1.2).astype(np.float32)
    n = 200_000
    x = np.broadcast_to(base, (n, 12))
    out = oracle.filter_softmax(x, "f32", 0.9, 8, 0.9, rng=(2024, 5), rows_per_request=4)
    ref = filtered_dist(base, 0.9, 8, 0.9)
    counts = np.bincount(out["sample"], minlength=12)
    assert chi2_pvalue(counts, ref) > 1e-4
    # changing the cycle changes the draws
    out2 = oracle.filter_softmax(x[:1000], "f32", 0.9, 8, 0.9, rng=(2024, 6), rows_per_request=4)
    assert not np.array_equal(out2["sample"], out["sample"][:1000])
