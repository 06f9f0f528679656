"""Pins of the oracle's two-pass cycle layout (linear mode).

The UNO PR page ("Motivation", "Modifications" and the review thread on the
token counters) and the evaluation guide (单模型双前向架构) describe a cycle
whose draft pass yields an exact base-weights first token plus B - 1
proposals, with B + 1 output slots per request and
num_correct_drafts = accept_len - 2.  The generic linear verification is this
layout's special case in which the first draft row and the first target row
are the same distribution (its first draft is then accepted with
probability 1), so the two written-out paths must emit the same tokens.
"""
import itertools

import numpy as np
import pytest

import oracle
from _defs import chi2_pvalue, filtered_dist
from test_oracle_linear import TinyAR
from test_oracle_params import _params


def _rows(R, B, vocab, seed, noise=0.4):
    """Draft and target logits [R, B, vocab]; target row i - 1, which
    verifies proposal i, is draft row i plus noise; the last target row (the
    bonus) is drawn afresh."""
    rng = np.random.default_rng(seed)
    draft = (rng.standard_normal((R, B, vocab)) * 1.5).astype(np.float32)
    target = np.empty_like(draft)
    target[:, :B - 1] = draft[:, 1:] + rng.standard_normal((R, B - 1, vocab)) * noise
    target[:, B - 1] = rng.standard_normal((R, vocab)) * 1.5
    return draft, target


def _generic(draft, target, R, B, T, K, P, rng, order):
    """The same cycle run through the generic verification: draft x_0 is
    verified against its own row, then x_i against target row i - 1."""
    vocab = draft.shape[-1]
    cap = max(1, min(int(np.max(K)), vocab))
    q = oracle.filter_softmax(draft.reshape(R * B, vocab), "f32", T, K, P, rows_per_request=B, cap=cap,
                              rng=rng, order=order)
    tgt = np.concatenate([draft[:, :1], target], axis=1).reshape(R * (B + 1), vocab)
    out = oracle.linear_verify(tgt, "f32", R, B, T, K, P, q["sample"].reshape(R, B), q["ids"], q["probs"],
                               q["count"], rng=rng, order=order)
    return q, out


@pytest.mark.parametrize("B,order,per_request", [(4, "topk_first", False), (4, "joint", True),
                                                  (1, "topk_first", True), (6, "joint", False)])
def test_cycle_equals_generic_form_with_a_certain_first_draft(B, order, per_request):
    R, vocab = 400, 60
    draft, target = _rows(R, B, vocab, 61 + B)
    if per_request:
        T, K, P = _params(R, 62)
    else:
        T, K, P = 0.9, 20, 0.9
    rng = (17, 2, 5)
    cyc = oracle.linear_cycle(draft.reshape(R * B, vocab), target.reshape(R * B, vocab), "f32", R, B, T, K, P,
                              rng, order=order)
    q, gen = _generic(draft, target, R, B, T, K, P, rng, order)
    assert np.all(gen["accept_len"] >= 1)  # the first draft is never rejected
    assert np.array_equal(cyc["tokens"], gen["tokens"])
    assert np.array_equal(cyc["accept_len"], gen["num_tokens"])
    assert np.array_equal(cyc["num_correct_drafts"], gen["accept_len"] - 1)
    assert np.array_equal(cyc["flags"], gen["flags"])
    # token 0 is the draw from the base-weights row, unconditionally
    assert np.array_equal(cyc["tokens"][:, 0], q["sample"].reshape(R, B)[:, 0])
    if B > 1:  # every proposal accepted (the bonus drawn) and some rejected
        assert 0.05 < np.mean(cyc["num_correct_drafts"] == B - 1) < 0.95


def test_cycle_counters_and_output_slots():
    R, B, vocab = 500, 5, 40
    draft, target = _rows(R, B, vocab, 63)
    out = oracle.linear_cycle(draft.reshape(R * B, vocab), target.reshape(R * B, vocab), "f32", R, B, 1.0, 30,
                              0.95, (9, 4))
    x = oracle.filter_softmax(draft.reshape(R * B, vocab), "f32", 1.0, 30, 0.95, rows_per_request=B,
                              rng=(9, 4))["sample"].reshape(R, B)
    acc, ncd, toks = out["accept_len"], out["num_correct_drafts"], out["tokens"]
    assert toks.shape == (R, B + 1)  # B + 1 output slots per request
    assert np.all(out["flags"] == 0)
    assert np.array_equal(ncd, acc - 2)  # two tokens of a cycle are not drafts
    assert np.all((ncd >= 0) & (ncd <= B - 1))
    for r in range(R):
        # token 0 and the accepted proposals are the drafts, in order
        assert np.array_equal(toks[r, :1 + ncd[r]], x[r, :1 + ncd[r]])
        assert np.all(toks[r, acc[r]:] == -1)
        assert np.all(toks[r, :acc[r]] >= 0)
    # the generated-token count of the batch: correct drafts plus two per request
    assert int(ncd.sum()) + 2 * R == int(acc.sum())


def test_single_row_cycle_is_first_token_plus_bonus():
    R, vocab = 40_000, 12
    rng = np.random.default_rng(64)
    d0 = (rng.standard_normal(vocab) * 1.3).astype(np.float32)
    t0 = (rng.standard_normal(vocab) * 1.3).astype(np.float32)
    draft = np.ascontiguousarray(np.broadcast_to(d0, (R, vocab)))
    target = np.ascontiguousarray(np.broadcast_to(t0, (R, vocab)))
    out = oracle.linear_cycle(draft, target, "f32", R, 1, 1.0, 12, 1.0, (5, 0))
    assert np.all(out["accept_len"] == 2) and np.all(out["num_correct_drafts"] == 0)
    assert chi2_pvalue(np.bincount(out["tokens"][:, 0], minlength=vocab), filtered_dist(d0, 1.0, 12, 1.0)) > 1e-4
    assert chi2_pvalue(np.bincount(out["tokens"][:, 1], minlength=vocab), filtered_dist(t0, 1.0, 12, 1.0)) > 1e-4


@pytest.mark.parametrize("vocab,B,T,k,p,order,seed", [(4, 3, 1.0, 4, 1.0, "topk_first", 71),
                                                      (5, 2, 0.8, 4, 0.9, "topk_first", 72),
                                                      (5, 2, 1.0, 3, 0.75, "joint", 52)])
def test_cycle_is_lossless(vocab, B, T, k, p, order, seed):
    """Token 0 follows the base-weights row (the target's own first
    distribution), and every later token the target given its prefix."""
    ar = TinyAR(vocab, B, seed)
    rng = np.random.default_rng(seed + 100)
    lora = (rng.standard_normal((B - 1, vocab)) * 1.5).astype(np.float32)
    R = 120_000
    draft = np.empty((R, B, vocab), dtype=np.float32)
    draft[:, 0] = ar.rows[()]
    draft[:, 1:] = lora
    draft = draft.reshape(R * B, vocab)
    x = oracle.filter_softmax(draft, "f32", T, k, p, rows_per_request=B, rng=(seed, 1),
                              order=order)["sample"].reshape(R, B)
    target = np.empty((R, B, vocab), dtype=np.float32)
    for r in range(R):
        for i in range(B):
            target[r, i] = ar.rows[tuple(x[r, :i + 1])]
    out = oracle.linear_cycle(draft, target.reshape(R * B, vocab), "f32", R, B, T, k, p, (seed, 1), order=order)
    toks, acc = out["tokens"], out["accept_len"]
    assert np.array_equal(toks[:, 0], x[:, 0])
    seqs = np.full((R, B + 1), -1, dtype=np.int64)
    for r in range(R):
        seqs[r, :acc[r]] = toks[r, :acc[r]]
    crng = np.random.default_rng(seed + 200)
    for t in range(B + 1):
        need = np.nonzero(seqs[:, t] < 0)[0]
        u = crng.random(need.size)
        for n, r in enumerate(need):
            d = ar.dist(seqs[r, :t], T, k, p, order)
            seqs[r, t] = min(int(np.searchsorted(np.cumsum(d), u[n] * d.sum(), side="right")), vocab - 1)
    codes = (seqs * (vocab ** np.arange(B + 1))).sum(axis=1)
    counts = np.bincount(codes, minlength=vocab ** (B + 1))
    probs = np.zeros(vocab ** (B + 1))
    for seq in itertools.product(range(vocab), repeat=B + 1):
        probs[int(np.dot(seq, vocab ** np.arange(B + 1)))] = ar.seq_prob(list(seq), T, k, p, order)
    assert chi2_pvalue(counts, probs) > 1e-4
    ncd = out["num_correct_drafts"]
    assert 0.05 < np.mean(ncd == B - 1) < 0.95 or 0.05 < np.mean(ncd == 0) < 0.95


def test_non_finite_rows():
    R, B, vocab = 4, 3, 20
    draft, target = _rows(R, B, vocab, 65)
    draft[0, 0, 5] = np.nan  # no base-weights token: nothing is emitted
    draft[1, 1, :] = -np.inf  # a proposal with no support: rejected, resampled from p
    target[2, 0, 3] = np.inf  # the row verifying proposal 1: the request stops there
    target[3, 2, 0] = np.nan  # a row the walk may not reach still flags the request
    out = oracle.linear_cycle(draft.reshape(R * B, vocab), target.reshape(R * B, vocab), "f32", R, B, 1.0, 10,
                              0.9, (2, 0))
    acc, ncd, toks, fl = out["accept_len"], out["num_correct_drafts"], out["tokens"], out["flags"]
    assert acc[0] == 0 and ncd[0] == 0 and np.all(toks[0] == -1) and fl[0] & oracle.FLAG_NONFINITE_ROW
    assert fl[1] & oracle.FLAG_NONFINITE_ROW and fl[1] & oracle.FLAG_DRAFT_NOT_IN_SUPPORT
    assert ncd[1] == 0 and acc[1] == 2 and toks[1, 1] >= 0  # rejected at proposal 1, token drawn from p
    assert acc[2] == 1 and ncd[2] == 0 and toks[2, 0] >= 0 and fl[2] & oracle.FLAG_NONFINITE_ROW
    assert fl[3] & oracle.FLAG_NONFINITE_ROW


def test_cycle_argument_errors():
    draft, target = _rows(2, 2, 8, 66)
    d, t = draft.reshape(4, 8), target.reshape(4, 8)
    with pytest.raises(oracle.OracleError):
        oracle.linear_cycle(d, t, "f32", 2, 2, 1.0, 0, 0.9, (1, 0))
    with pytest.raises(oracle.OracleError):
        oracle.linear_cycle(d, t, "f32", 2, 2, [1.0, -1.0], 4, 0.9, (1, 0))
    with pytest.raises(ValueError):
        oracle.linear_cycle(d, t, "f32", 2, 2, 1.0, 4, 0.9, (1, 0), order="dense")
    # zero requests is a valid, empty call
    e = np.zeros((0, 8), np.float32)
    out = oracle.linear_cycle(e, e, "f32", 0, 2, 1.0, 4, 0.9, (1, 0))
    assert out["tokens"].shape == (0, 3)
