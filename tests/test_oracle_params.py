"""Pins of the oracle's per-request sampling parameters and of the "joint"
filter order.

The UNO PR page's review thread on the filter order contrasts UNO's order
(top-k, renormalise, then top-p) with the regular sampler's joint order, in
which top-p is computed from the full softmax.  The joint order is pinned by a
worked example derived by hand, by the closed form of a geometric row, and by
its definition written with library routines; per-request parameters are
pinned by reduction to separate single-request calls.
"""
import itertools

import numpy as np
import pytest

import oracle
from _defs import chi2_pvalue, filtered_dist, top_p_margin
from test_oracle_linear import TinyAR


def _compact(out, r):
    c = out["count"][r]
    return {int(i): float(p) for i, p in zip(out["ids"][r, :c], out["probs"][r, :c])}


# Logits ln 4, ln 2, 0, 0 give weights 4 : 2 : 1 : 1, so the full softmax is
# 1/2, 1/4, 1/8, 1/8; ids 2 and 3 tie and id 2 ranks first.  At T = 2 the
# weights are 2 : sqrt2 : 1 : 1.
_S2 = np.sqrt(2.0)
WORKED = [
    # T, top_k, top_p, top-k-first result, joint result
    # top-2 renormalised is 2/3, 1/3: the mass before id 1 is 2/3 >= 0.6, id 0
    # alone; the full-softmax mass before id 1 is 1/2 < 0.6, ids 0 and 1.
    (1.0, 2, 0.6, {0: 1.0}, {0: 2 / 3, 1: 1 / 3}),
    # top-3 renormalised is 4/7, 2/7, 1/7: masses before ids 1, 2 are 4/7 and
    # 6/7, so ids 0, 1; full-softmax masses before are 1/2 and 3/4 < 0.8, so
    # ids 0, 1, 2.
    (1.0, 3, 0.8, {0: 2 / 3, 1: 1 / 3}, {0: 4 / 7, 1: 2 / 7, 2: 1 / 7}),
    # top_k = vocab: both orders read the same masses, 1/2 and 3/4 >= 0.7.
    (1.0, 4, 0.7, {0: 2 / 3, 1: 1 / 3}, {0: 2 / 3, 1: 1 / 3}),
    # T = 2, top-2 renormalised: 2 / (2 + sqrt2) = 0.586 >= 0.45, id 0 alone;
    # full softmax: 2 / (4 + sqrt2) = 0.369 < 0.45, ids 0 and 1.
    (2.0, 2, 0.45, {0: 1.0}, {0: 2 / (2 + _S2), 1: _S2 / (2 + _S2)}),
    # top_p = 1 keeps the top-k in both orders.
    (1.0, 3, 1.0, {0: 4 / 7, 1: 2 / 7, 2: 1 / 7}, {0: 4 / 7, 1: 2 / 7, 2: 1 / 7}),
]


@pytest.mark.parametrize("T,k,p,first,joint", WORKED)
def test_joint_order_worked_example(T, k, p, first, joint):
    x = np.array([[np.log(4.0), np.log(2.0), 0.0, 0.0]], dtype=np.float32)
    for order, expect in (("topk_first", first), ("joint", joint)):
        got = _compact(oracle.filter_softmax(x, "f32", T, k, p, cap=4, order=order), 0)
        assert sorted(got) == sorted(expect), (order, got, expect)
        for i in expect:
            assert abs(got[i] - expect[i]) < 1e-6, (order, got, expect)


@pytest.mark.parametrize("N,T", [(10, 1.0), (37, 1.0), (24, 2.5), (60, 0.6)])
def test_geometric_row_closed_form(N, T):
    # l_j = -j: softmax(l / T)_j is proportional to r^j with r = exp(-1/T), and
    # the first j of a set of n such tokens hold (1 - r^j) / (1 - r^n) of its
    # mass (a finite geometric series).  The set is the top-k under the
    # top-k-first order and the whole row under the joint order.
    x = (-np.arange(N, dtype=np.float64)).astype(np.float32)[None, :]
    r = np.exp(-1.0 / float(np.float32(T)))  # the call passes T as binary32
    checked = 0
    for k in (1, 2, 3, 5, 8, N):
        for p in (0.3, 0.55, 0.7, 0.8, 0.9, 0.97, 0.999):
            for order, n in (("topk_first", min(k, N)), ("joint", N)):
                before = [(1 - r ** j) / (1 - r ** n) for j in range(1, min(k, N))]
                if any(abs(b - p) < 1e-6 for b in before):
                    continue
                L = 1 + sum(b < p for b in before)  # the masses before rise with j
                out = oracle.filter_softmax(x, "f32", T, k, p, cap=N, order=order)
                assert out["count"][0] == L, (k, p, order)
                assert np.array_equal(out["ids"][0, :L], np.arange(L))
                expect = r ** np.arange(L) * (1 - r) / (1 - r ** L)
                np.testing.assert_allclose(out["probs"][0, :L], expect, rtol=2e-7, atol=1e-12)
                checked += 1
    assert checked > 75  # of 6 x 7 x 2 cases; those within 1e-6 of a cut are skipped


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,k,p", [(1.0, 50, 0.95), (0.7, 20, 0.9), (1.3, 100, 0.5), (1.0, 5, 0.3)])
def test_joint_matches_library_definition(dtype, T, k, p):
    rng = np.random.default_rng(41)
    x = (rng.standard_normal((150, 400)) * 1.5).astype(np.float32)
    x[:, 17] += 4.0  # a dominant token, as in sharp decoding distributions
    if dtype == "bf16":
        bits = (x.view(np.uint32) >> 16).astype(np.uint16)
        x = (bits.astype(np.uint32) << 16).view(np.float32)
        arg = bits
    else:
        arg = x
    out = oracle.filter_softmax(arg, dtype, T, k, p, dense=True, order="joint")
    checked = 0
    for r in range(x.shape[0]):
        if top_p_margin(x[r], T, k, p, "joint") < 1e-9:
            continue
        ref = filtered_dist(x[r], T, k, p, "joint")
        assert out["count"][r] == np.count_nonzero(ref)
        assert np.max(np.abs(out["dense"][r] - ref)) < 1e-7
        checked += 1
    assert checked > 140


def test_joint_support_nests_and_reduces():
    rng = np.random.default_rng(42)
    x = (rng.standard_normal((120, 300)) * 2).astype(np.float32)
    grew = 0
    for T, k, p in [(1.0, 50, 0.95), (0.8, 30, 0.8), (1.5, 200, 0.9), (1.0, 10, 0.5)]:
        a = oracle.filter_softmax(x, "f32", T, k, p, dense=True)
        b = oracle.filter_softmax(x, "f32", T, k, p, dense=True, order="joint")
        sa, sb = a["dense"] > 0, b["dense"] > 0
        # a full-softmax prefix mass never exceeds the renormalised one, so the
        # joint cut keeps at least the top-k-first support, within the top-k
        assert np.all(sa <= sb)
        assert np.all(b["count"] <= min(k, x.shape[1]))
        grew += int(np.sum(b["count"] > a["count"]))
    assert grew > 50
    # top_p = 1, or top_k at least the vocabulary, leaves nothing to differ
    for T, k, p in [(1.0, 50, 1.0), (0.7, 300, 0.9), (1.2, 400, 0.6)]:
        a = oracle.filter_softmax(x, "f32", T, k, p, cap=300, dense=True, rng=(3, 1))
        b = oracle.filter_softmax(x, "f32", T, k, p, cap=300, dense=True, rng=(3, 1), order="joint")
        for key in ("ids", "probs", "count", "dense", "sample"):
            assert np.array_equal(a[key], b[key]), key


def test_joint_draw_follows_the_filtered_distribution():
    rng = np.random.default_rng(43)
    row = (rng.standard_normal(60) * 1.2).astype(np.float32)
    R = 60_000
    x = np.ascontiguousarray(np.broadcast_to(row, (R, 60)))
    out = oracle.filter_softmax(x, "f32", 0.9, 25, 0.85, rng=(8, 0), order="joint")
    ref = filtered_dist(row, 0.9, 25, 0.85, "joint")
    assert chi2_pvalue(np.bincount(out["sample"], minlength=60), ref) > 1e-4
    assert not np.allclose(ref, filtered_dist(row, 0.9, 25, 0.85))  # the orders differ on this row


def _params(nreq, seed):
    rng = np.random.default_rng(seed)
    T = rng.choice([0.0, 0.6, 1.0, 1.4], size=nreq).astype(np.float32)
    K = rng.choice([1, 7, 20, 90], size=nreq).astype(np.int32)
    P = rng.choice([0.5, 0.9, 1.0], size=nreq).astype(np.float32)
    return T, K, P


@pytest.mark.parametrize("order", ["topk_first", "joint"])
def test_per_request_filter_equals_separate_calls(order):
    nreq, rpr, vocab = 7, 3, 90
    rng = np.random.default_rng(44)
    x = (rng.standard_normal((nreq * rpr - 1, vocab)) * 1.5).astype(np.float32)  # ragged last request
    T, K, P = _params(nreq, 45)
    whole = oracle.filter_softmax(x, "f32", T, K, P, rows_per_request=rpr, cap=vocab, rng=(6, 2, 10),
                                  dense=True, order=order)
    for q in range(nreq):
        rows = slice(q * rpr, min((q + 1) * rpr, x.shape[0]))
        one = oracle.filter_softmax(x[rows], "f32", float(T[q]), int(K[q]), float(P[q]),
                                    rows_per_request=rpr, cap=vocab, rng=(6, 2, 10 + q), dense=True,
                                    order=order)
        for key in ("ids", "probs", "count", "flags", "dense", "sample", "margin"):
            assert np.array_equal(whole[key][rows], one[key]), (q, key)


@pytest.mark.parametrize("order", ["topk_first", "joint"])
def test_per_request_linear_verify_equals_separate_calls(order):
    R, B, vocab = 8, 3, 50
    rng = np.random.default_rng(46)
    g = (rng.standard_normal((R, B + 1, vocab)) * 1.5).astype(np.float32)
    T, K, P = _params(R, 47)
    q = oracle.filter_softmax(g[:, :B].reshape(R * B, vocab), "f32", T, K, P, rows_per_request=B, cap=vocab,
                              rng=(2, 0), order=order)
    tgt = (g + rng.standard_normal(g.shape).astype(np.float32) * 0.7).reshape(R * (B + 1), vocab)
    drafts = q["sample"].reshape(R, B)
    whole = oracle.linear_verify(tgt, "f32", R, B, T, K, P, drafts, q["ids"], q["probs"], q["count"],
                                 rng=(2, 0, 4), order=order)
    for r in range(R):
        rows = slice(r * B, (r + 1) * B)
        one = oracle.linear_verify(tgt[r * (B + 1):(r + 1) * (B + 1)], "f32", 1, B, float(T[r]), int(K[r]),
                                   float(P[r]), drafts[r:r + 1], q["ids"][rows], q["probs"][rows],
                                   q["count"][rows], rng=(2, 0, 4 + r), order=order)
        for key in whole:
            assert np.array_equal(whole[key][r:r + 1], one[key]), (r, key)


@pytest.mark.parametrize("order", ["topk_first", "joint"])
def test_per_request_tree_verify_equals_separate_calls(order):
    R, B, V, vocab = 6, 2, 5, 40
    rng = np.random.default_rng(48)
    tgt = (rng.standard_normal((R * V, vocab)) * 1.5).astype(np.float32)
    T, K, P = _params(R, 49)
    tk = np.tile(np.array([-1, 3, 7, 3, 1], np.int32), (R, 1))
    pa = np.tile(np.array([-1, 0, 0, 1, 1], np.int32), (R, 1))
    nn = np.full(R, V, np.int32)
    whole = oracle.tree_verify(tgt, "f32", R, B, V, T, K, P, tk, pa, nn, rng=(3, 1, 2), order=order)
    for r in range(R):
        one = oracle.tree_verify(tgt[r * V:(r + 1) * V], "f32", 1, B, V, float(T[r]), int(K[r]), float(P[r]),
                                 tk[r:r + 1], pa[r:r + 1], nn[r:r + 1], rng=(3, 1, 2 + r), order=order)
        for key in whole:
            assert np.array_equal(whole[key][r:r + 1], one[key]), (r, key)


@pytest.mark.parametrize("vocab,B,T,k,p,seed", [(4, 2, 1.0, 2, 0.75, 53), (5, 2, 1.0, 3, 0.75, 52)])
def test_joint_linear_output_is_the_joint_target_process(vocab, B, T, k, p, seed):
    ar = TinyAR(vocab, B, seed)
    rng = np.random.default_rng(seed + 100)
    q_logits = (rng.standard_normal((B, vocab)) * 1.5).astype(np.float32)
    R = 100_000
    xq = np.ascontiguousarray(np.broadcast_to(q_logits, (R, B, vocab)).reshape(R * B, vocab))
    q = oracle.filter_softmax(xq, "f32", T, k, p, rows_per_request=B, rng=(seed, 3), order="joint")
    drafts = q["sample"].reshape(R, B)
    target = np.empty((R, B + 1, vocab), dtype=np.float32)
    for r in range(R):
        for i in range(B + 1):
            target[r, i] = ar.rows[tuple(drafts[r, :i])]
    out = oracle.linear_verify(target.reshape(R * (B + 1), vocab), "f32", R, B, T, k, p, drafts, q["ids"],
                               q["probs"], q["count"], rng=(seed, 3), order="joint")
    toks, ntok = out["tokens"], out["num_tokens"]
    seqs = np.full((R, B + 1), -1, dtype=np.int64)
    for r in range(R):
        seqs[r, :ntok[r]] = toks[r, :ntok[r]]
    crng = np.random.default_rng(seed + 200)
    for t in range(B + 1):
        need = np.nonzero(seqs[:, t] < 0)[0]
        u = crng.random(need.size)
        for n, r in enumerate(need):
            d = ar.dist(seqs[r, :t], T, k, p, "joint")
            seqs[r, t] = min(int(np.searchsorted(np.cumsum(d), u[n] * d.sum(), side="right")), vocab - 1)
    codes = (seqs * (vocab ** np.arange(B + 1))).sum(axis=1)
    counts = np.bincount(codes, minlength=vocab ** (B + 1))
    probs = np.zeros(vocab ** (B + 1))
    joint_differs = False
    for seq in itertools.product(range(vocab), repeat=B + 1):
        code = int(np.dot(seq, vocab ** np.arange(B + 1)))
        probs[code] = ar.seq_prob(list(seq), T, k, p, "joint")
        joint_differs |= abs(probs[code] - ar.seq_prob(list(seq), T, k, p)) > 1e-3
    assert joint_differs  # the case separates the two orders
    assert chi2_pvalue(counts, probs) > 1e-4


def test_joint_tree_root_draw_follows_the_joint_filter():
    # V = B = 1: the tree is the root alone and the emitted token is the
    # root row's draw
    R, vocab = 50_000, 30
    rng = np.random.default_rng(53)
    row = (rng.standard_normal(vocab) * 1.3).astype(np.float32)
    tgt = np.ascontiguousarray(np.broadcast_to(row, (R, vocab)))
    tk = np.full((R, 1), -1, np.int32)
    out = oracle.tree_verify(tgt, "f32", R, 1, 1, 1.0, 12, 0.7, tk, tk, np.ones(R, np.int32), rng=(4, 0),
                             order="joint")
    assert np.all(out["num_tokens"] == 1)
    ref = filtered_dist(row, 1.0, 12, 0.7, "joint")
    assert not np.allclose(ref, filtered_dist(row, 1.0, 12, 0.7))
    assert chi2_pvalue(np.bincount(out["tokens"][:, 0], minlength=vocab), ref) > 1e-4


def test_per_request_parameter_errors():
    x = np.zeros((4, 10), np.float32)
    for T, K, P in [([1.0, -1.0], 5, 0.9), (1.0, [5, 0], 0.9), (1.0, 5, [0.9, 1.5]), (1.0, 5, [0.0, 0.9])]:
        with pytest.raises(oracle.OracleError):
            oracle.filter_softmax(x, "f32", T, K, P, rows_per_request=2, cap=10)
    with pytest.raises(ValueError):
        oracle.filter_softmax(x, "f32", 1.0, 5, 0.9, order="dense")
    # cap must hold the widest request
    with pytest.raises(oracle.OracleError):
        oracle.filter_softmax(x, "f32", 1.0, [3, 8], 0.9, rows_per_request=2, cap=5)
