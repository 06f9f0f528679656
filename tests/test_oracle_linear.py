"""Pins of the oracle's linear-mode rejection sampling.

The method is lossless (UNO PR page, "Motivation"): whatever the draft
marginals, the emitted tokens must follow the target-only autoregressive
process.  A tiny vocabulary with a prefix-dependent target table makes that
checkable by a chi-square test over every sequence of length B+1.
"""
import itertools

import numpy as np
import pytest

import oracle
from _defs import chi2_pvalue, filtered_dist


class TinyAR:
    """A table of target logits for every prefix of length 0..B."""

    def __init__(self, vocab, B, seed, scale=1.5):
        rng = np.random.default_rng(seed)
        self.vocab, self.B = vocab, B
        self.rows = {}
        for L in range(B + 1):
            for pre in itertools.product(range(vocab), repeat=L):
                self.rows[pre] = (rng.standard_normal(vocab) * scale).astype(np.float32)

    def dist(self, prefix, T, k, p, order="topk_first"):
        return filtered_dist(self.rows[tuple(prefix)], T, k, p, order)

    def seq_prob(self, seq, T, k, p, order="topk_first"):
        pr = 1.0
        for t in range(len(seq)):
            pr *= self.dist(seq[:t], T, k, p, order)[seq[t]]
        return pr


def _propose(q_logits, R, B, T, k, p, rng):
    x = np.ascontiguousarray(np.broadcast_to(q_logits, (R, B, q_logits.shape[-1])).reshape(R * B, -1))
    out = oracle.filter_softmax(x, "f32", T, k, p, rows_per_request=B, rng=rng)
    return out["sample"].reshape(R, B), out


def _complete(ar, emitted, B, T, k, p, rng):
    """Extend each emitted prefix to B+1 tokens by sampling the target process."""
    R = len(emitted)
    seqs = np.full((R, B + 1), -1, dtype=np.int64)
    for r, e in enumerate(emitted):
        seqs[r, :len(e)] = e
    for t in range(B + 1):
        need = np.nonzero(seqs[:, t] < 0)[0]
        if need.size == 0:
            continue
        u = rng.random(need.size)
        for n, r in enumerate(need):
            d = ar.dist(seqs[r, :t], T, k, p)
            seqs[r, t] = min(int(np.searchsorted(np.cumsum(d), u[n] * d.sum(), side="right")), ar.vocab - 1)
    return seqs


@pytest.mark.parametrize("vocab,B,T,k,p,seed", [(4, 2, 1.0, 4, 1.0, 11), (5, 2, 0.8, 4, 0.9, 12),
                                                (3, 3, 1.2, 3, 0.95, 13)])
def test_linear_output_is_the_target_process(vocab, B, T, k, p, seed):
    ar = TinyAR(vocab, B, seed)
    rng = np.random.default_rng(seed + 100)
    q_logits = (rng.standard_normal((B, vocab)) * 1.5).astype(np.float32)
    R = 120_000
    drafts, q = _propose(q_logits, R, B, T, k, p, rng=(seed, 3))
    target = np.empty((R, B + 1, vocab), dtype=np.float32)
    for r in range(R):
        for i in range(B + 1):
            target[r, i] = ar.rows[tuple(drafts[r, :i])]
    out = oracle.linear_verify(target.reshape(R * (B + 1), vocab), "f32", R, B, T, k, p, drafts,
                               q["ids"], q["probs"], q["count"], rng=(seed, 3))
    acc, ntok, toks = out["accept_len"], out["num_tokens"], out["tokens"]
    assert np.all((acc >= 0) & (acc <= B)) and np.array_equal(ntok, acc + 1)
    for r in range(200):
        assert np.array_equal(toks[r, :acc[r]], drafts[r, :acc[r]])
        assert np.all(toks[r, ntok[r]:] == -1)
    emitted = [toks[r, :ntok[r]] for r in range(R)]
    seqs = _complete(ar, emitted, B, T, k, p, np.random.default_rng(seed + 200))
    codes = (seqs * (vocab ** np.arange(B + 1))).sum(axis=1)
    counts = np.bincount(codes, minlength=vocab ** (B + 1))
    probs = np.zeros(vocab ** (B + 1))
    for seq in itertools.product(range(vocab), repeat=B + 1):
        probs[int(np.dot(seq, vocab ** np.arange(B + 1)))] = ar.seq_prob(list(seq), T, k, p)
    assert chi2_pvalue(counts, probs) > 1e-4
    # and the drafts are not trivially always accepted or always rejected
    assert 0.05 < np.mean(acc == B) < 0.95 or 0.05 < np.mean(acc == 0) < 0.95


def test_mean_accept_length_closed_form():
    vocab, B, T, k, p = 30, 5, 1.0, 20, 0.95
    rng = np.random.default_rng(21)
    g = (rng.standard_normal((B + 1, vocab)) * 1.3).astype(np.float32)
    q_logits = g[:B]
    p_logits = (g + rng.standard_normal(g.shape) * 0.8).astype(np.float32)
    R = 100_000
    drafts, q = _propose(q_logits, R, B, T, k, p, rng=(5, 0))
    target = np.ascontiguousarray(np.broadcast_to(p_logits, (R, B + 1, vocab)).reshape(-1, vocab))
    out = oracle.linear_verify(target, "f32", R, B, T, k, p, drafts, q["ids"], q["probs"], q["count"],
                               rng=(5, 0))
    alpha = [np.minimum(filtered_dist(p_logits[i], T, k, p), filtered_dist(q_logits[i], T, k, p)).sum()
             for i in range(B)]
    expect = sum(np.prod(alpha[:m]) for m in range(1, B + 1))
    acc = out["accept_len"].astype(np.float64)
    assert abs(acc.mean() - expect) < 4 * acc.std() / np.sqrt(R)
    # acceptance at position i given it was reached is alpha_i
    for i in range(B):
        reached = acc >= i
        rate = np.mean(acc[reached] > i)
        assert abs(rate - alpha[i]) < 4 * np.sqrt(alpha[i] * (1 - alpha[i]) / reached.sum()) + 1e-9


def test_equal_draft_and_target_accept_everything():
    vocab, B, R = 50, 6, 2000
    rng = np.random.default_rng(22)
    g = rng.standard_normal((B + 1, vocab)).astype(np.float32)
    drafts, q = _propose(g[:B], R, B, 1.0, 20, 0.9, rng=(9, 1))
    target = np.ascontiguousarray(np.broadcast_to(g, (R, B + 1, vocab)).reshape(-1, vocab))
    out = oracle.linear_verify(target, "f32", R, B, 1.0, 20, 0.9, drafts, q["ids"], q["probs"], q["count"],
                               rng=(9, 1))
    assert np.all(out["accept_len"] == B)
    assert np.array_equal(out["tokens"][:, :B], drafts)
    bonus = out["tokens"][:, B]
    assert chi2_pvalue(np.bincount(bonus, minlength=vocab), filtered_dist(g[B], 1.0, 20, 0.9)) > 1e-4


def test_disjoint_one_hot_rejects_at_first_position():
    vocab, B, R = 16, 4, 50
    rng = np.random.default_rng(23)
    q_logits = rng.standard_normal((B, vocab)).astype(np.float32)
    p_logits = rng.standard_normal((B + 1, vocab)).astype(np.float32)
    q_logits[0, :] = 0
    q_logits[0, 3] = 5
    p_logits[0, :] = 0
    p_logits[0, 9] = 5
    drafts, q = _propose(q_logits, R, B, 1.0, 1, 1.0, rng=(1, 0))
    target = np.ascontiguousarray(np.broadcast_to(p_logits, (R, B + 1, vocab)).reshape(-1, vocab))
    out = oracle.linear_verify(target, "f32", R, B, 1.0, 1, 1.0, drafts, q["ids"], q["probs"], q["count"],
                               rng=(1, 0))
    assert np.all(out["accept_len"] == 0)
    assert np.all(out["tokens"][:, 0] == 9)
    assert np.all(out["num_tokens"] == 1)


def test_top_k_one_is_greedy_speculative_decoding():
    vocab, B, R = 40, 6, 300
    rng = np.random.default_rng(24)
    q_logits = rng.integers(0, 3, size=(R, B, vocab)).astype(np.float32)
    p_logits = rng.integers(0, 3, size=(R, B + 1, vocab)).astype(np.float32)
    out_q = oracle.filter_softmax(q_logits.reshape(-1, vocab), "f32", 1.0, 1, 1.0, rows_per_request=B,
                                  rng=(3, 0))
    drafts = out_q["sample"].reshape(R, B)
    out = oracle.linear_verify(p_logits.reshape(-1, vocab), "f32", R, B, 1.0, 1, 1.0, drafts, out_q["ids"],
                               out_q["probs"], out_q["count"], rng=(3, 0))
    g = np.argmax(p_logits, axis=2)
    for r in range(R):
        m = 0
        while m < B and drafts[r, m] == g[r, m]:
            m += 1
        assert out["accept_len"][r] == m
        assert np.array_equal(out["tokens"][r, :m + 1], np.append(drafts[r, :m], g[r, m]))


def test_draft_outside_support_is_rejected_and_flagged():
    vocab, B = 20, 3
    rng = np.random.default_rng(25)
    g = rng.standard_normal((B + 1, vocab)).astype(np.float32)
    q = oracle.filter_softmax(g[:B], "f32", 1.0, 5, 1.0, rows_per_request=B, rng=(2, 0))
    drafts = q["sample"].reshape(1, B).copy()
    outside = [t for t in range(vocab) if t not in set(q["ids"][0, :q["count"][0]])][0]
    drafts[0, 0] = outside
    out = oracle.linear_verify(g, "f32", 1, B, 1.0, 5, 1.0, drafts, q["ids"], q["probs"], q["count"],
                               rng=(2, 0))
    assert out["accept_len"][0] == 0
    assert out["flags"][0] & oracle.FLAG_DRAFT_NOT_IN_SUPPORT


def test_non_finite_target_row_stops_the_request():
    vocab, B = 20, 3
    g = np.tile(np.linspace(0, 1, vocab, dtype=np.float32), (B + 1, 1))
    q = oracle.filter_softmax(g[:B], "f32", 1.0, 5, 1.0, rows_per_request=B, rng=(2, 0))
    drafts = q["sample"].reshape(1, B)
    tgt = g.copy()
    tgt[2, 4] = np.nan
    out = oracle.linear_verify(tgt, "f32", 1, B, 1.0, 5, 1.0, drafts, q["ids"], q["probs"], q["count"],
                               rng=(2, 0))
    # rows 0 and 1 equal the draft rows, so both drafts are accepted; row 2 is NaN
    assert out["accept_len"][0] == 2 and out["num_tokens"][0] == 2
    assert out["tokens"][0, 2] == -1
    assert out["flags"][0] & oracle.FLAG_NONFINITE_ROW
