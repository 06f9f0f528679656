"""Exact enumeration of the oracle's output distribution on tiny vocabularies.

UNO is lossless like speculative decoding (UNO PR page, "Motivation"): the
tokens a cycle emits, completed to B + 1 tokens by the target process, are
distributed exactly as the target-only autoregressive (AR) process.  The
chi-square tests elsewhere check this by sampling; here it is checked exactly.

How.  Every decision of the oracle takes its uniform from one function, and a
test hook (``oracle.injected_uniforms``) lets the test choose those uniforms.
Each decision is a monotone step function of its uniform: the proposal draw
and every inverse-CDF draw pick a token that rises with u, and the accept test
holds for u below a threshold.  Bisection on the 53-bit grid the uniform lives
on (u = m * 2^-53) therefore finds, from the oracle's own code, the exact
probability of every branch: each proposal token, the accept test at every
position for every draft vector, each residual token after a rejection, and
each bonus token.  Summing over all draft vectors gives the exact output
distribution, which must equal prod_t p(s_t | s_<t) within 1e-12.  The tree
walk is enumerated the same way, node by node.

Rows are chosen so that every filtered probability is an exact binary
fraction c / 64 and every row sums to exactly 1 in binary32: then the
probabilities the oracle stores are the exact ones and losslessness holds to
rounding.  (With binary32 rows whose sums are off by an ulp, the identity
holds only to about 1e-7, which would hide small mistakes.)  The expected
target values come from the construction (c / 64), not from the oracle.
"""
import itertools

import numpy as np
import pytest

import oracle
from _defs import chi2_pvalue

GRID = 1 << 53  # uniforms are m * 2^-53, 0 <= m < 2^53
DEN = 64        # every kept weight is an integer, the kept weights of a row sum to DEN
F32 = "f32"


# ---------------------------------------------------------------------------
# Rows with exactly representable filtered probabilities.
# ---------------------------------------------------------------------------
def _candidate(rng, vocab, top_k, top_p, min_kept=1):
    """Logits (binary32) and the intended filtered weights c (integers summing
    to DEN) of one row: kk kept tokens with weights >= 2, possibly one extra
    token with weight 1/2 that the filter must cut (by top-k when kk reaches
    top_k, else by top-p < 1), the rest masked (-inf).  Kept tokens come from
    the first top_k + 1 ids, so that the supports of different rows overlap
    (drafts are then accepted and rejected with nontrivial probabilities)."""
    kk = int(rng.integers(min(min_kept, top_k, vocab), min(top_k, vocab) + 1))
    pool = min(vocab, top_k + 1)
    # a random composition of DEN into kk parts >= 2
    cuts = np.sort(rng.choice(np.arange(1, DEN // 2), size=kk - 1, replace=False)) if kk > 1 else np.array([], int)
    parts = np.diff(np.concatenate([[0], cuts, [DEN // 2]])) * 2
    toks = np.concatenate([rng.permutation(pool), pool + rng.permutation(vocab - pool)])
    kept = toks[:kk]
    c = np.zeros(vocab, dtype=np.int64)
    c[kept] = parts
    logits = np.full(vocab, -np.inf, dtype=np.float32)
    logits[kept] = np.log(parts.astype(np.float64)).astype(np.float32)
    extra_ok = kk < vocab and (kk >= top_k or top_p < 1.0)
    if extra_ok and rng.random() < 0.6:
        logits[toks[kk]] = np.float32(np.log(0.5))
    return logits, c


def dyadic_rows(n, vocab, top_k, top_p, seed, min_kept=1):
    """n rows whose filtered binary32 probabilities the oracle returns exactly
    as c / DEN (chosen by search: the binary32 logits log(c) are inexact, so
    only some candidates round back to c / DEN exactly)."""
    rng = np.random.default_rng(seed)
    rows, weights = [], []
    while len(rows) < n:
        cands = [_candidate(rng, vocab, top_k, top_p, min_kept) for _ in range(256)]
        L = np.stack([x[0] for x in cands])
        out = oracle.filter_softmax(L, F32, 1.0, top_k, top_p, cap=vocab)
        dense = np.zeros((len(cands), vocab))
        for r in range(len(cands)):
            cnt = out["count"][r]
            dense[r, out["ids"][r, :cnt]] = out["probs"][r, :cnt].astype(np.float64)
        for r, (lg, c) in enumerate(cands):
            if np.array_equal(dense[r], c / DEN) and len(rows) < n:
                rows.append(lg)
                weights.append(c / DEN)
    return np.stack(rows), np.stack(weights)


class DyadicAR:
    """Target logits for every prefix of length 0..B, each a dyadic row."""

    def __init__(self, vocab, B, top_k, top_p, seed):
        prefixes = [pre for L in range(B + 1) for pre in itertools.product(range(vocab), repeat=L)]
        rows, w = dyadic_rows(len(prefixes), vocab, top_k, top_p, seed)
        self.rows = {pre: rows[i] for i, pre in enumerate(prefixes)}
        self.w = {pre: w[i] for i, pre in enumerate(prefixes)}
        self.vocab, self.B = vocab, B

    def seq_prob(self, seq):
        pr = 1.0
        for t in range(len(seq)):
            pr *= self.w[tuple(seq[:t])][seq[t]]
        return pr


# ---------------------------------------------------------------------------
# Bisection on the uniform's grid, many queries at once.
# ---------------------------------------------------------------------------
def count_below(pred, nq):
    """For nq monotone predicates (true for small u), the number of grid points
    m in [0, 2^53) with pred(m * 2^-53) true.  pred(m) takes an int64 array of
    grid points (one per query) and returns a bool array."""
    lo = np.zeros(nq, dtype=np.int64)           # pred(lo) true, or lo == 0
    hi = np.full(nq, GRID, dtype=np.int64)      # pred(hi) false (hi == GRID: u = 1 counts as false)
    first = pred(lo)
    res = np.where(first, -1, 0)                # 0: pred false already at m = 0
    active = first.copy()
    while np.any(active & (hi - lo > 1)):
        mid = lo + (hi - lo) // 2
        mid = np.where(active, mid, lo)
        ok = pred(mid)
        lo = np.where(active & ok, mid, lo)
        hi = np.where(active & ~ok, mid, hi)
    return np.where(res == 0, 0, hi)


def u_of(m):
    return m.astype(np.float64) * (1.0 / GRID)


# ---------------------------------------------------------------------------
# Linear verification.
# ---------------------------------------------------------------------------
def _proposal_probs(q_logits, B, vocab, top_k, top_p):
    """P(x_i = t) of the oracle's proposal draw, per row i (exact)."""
    nq = B * vocab  # query (i, t): row i of request t... one request per boundary t

    def below(m):  # request t, row i: is the sample <= t at u_prop[t, i] = u(m)?
        table = np.zeros((vocab, B, 4))
        table[:, :, oracle.DRAW_PROPOSAL] = u_of(m).reshape(vocab, B)
        x = np.ascontiguousarray(np.broadcast_to(q_logits, (vocab, B, vocab)).reshape(vocab * B, vocab))
        with oracle.injected_uniforms(table):
            out = oracle.filter_softmax(x, F32, 1.0, top_k, top_p, rows_per_request=B, rng=(0, 0), cap=vocab)
        s = out["sample"].reshape(vocab, B)
        return (s <= np.arange(vocab)[:, None]).reshape(-1)

    C = count_below(below, nq).reshape(vocab, B).T  # C[i, t] = #u with sample <= t
    P = np.diff(np.concatenate([np.zeros((B, 1), np.int64), C], axis=1), axis=1)
    return P.astype(np.float64) / GRID


def _verify(ar, q, drafts, table, B):
    """Run the oracle's linear verification for one request per draft row."""
    R = len(drafts)
    target = np.stack([np.stack([ar.rows[tuple(x[:i])] for i in range(B + 1)]) for x in drafts])
    qi = np.broadcast_to(q["ids"][None], (R,) + q["ids"].shape).reshape(R * B, -1)
    qp = np.broadcast_to(q["probs"][None], (R,) + q["probs"].shape).reshape(R * B, -1)
    qc = np.broadcast_to(q["count"][None], (R, B)).reshape(-1)
    with oracle.injected_uniforms(table):
        return oracle.linear_verify(target.reshape(R * (B + 1), -1), F32, R, B, 1.0, ar.top_k, ar.top_p,
                                    np.asarray(drafts, dtype=np.int32), np.ascontiguousarray(qi),
                                    np.ascontiguousarray(qp), np.ascontiguousarray(qc), rng=(0, 0))


def linear_exact(vocab, B, top_k, top_p, seed):
    """Exact distribution of the oracle's completed linear output over the
    vocab^(B+1) sequences, and the AR table."""
    ar = DyadicAR(vocab, B, top_k, top_p, seed)
    ar.top_k, ar.top_p = top_k, top_p
    q_logits, _ = dyadic_rows(B, vocab, top_k, top_p, seed + 1000, min_kept=3)
    q = oracle.filter_softmax(q_logits, F32, 1.0, top_k, top_p, rows_per_request=B)
    Pq = _proposal_probs(q_logits, B, vocab, top_k, top_p)
    X = [x for x in itertools.product(range(vocab), repeat=B) if all(Pq[i, x[i]] > 0 for i in range(B))]
    nx = len(X)

    # accept thresholds theta[x, i]: earlier positions forced to accept (u = 0)
    def acc_pred(m):
        table = np.zeros((nx * B, B + 1, 4))
        table[:, :, oracle.DRAW_RESIDUAL] = 0.5
        table[:, :, oracle.DRAW_TARGET] = 0.5
        for i in range(B):
            table[i::B, i, oracle.DRAW_ACCEPT] = u_of(m[i::B])
        out = _verify(ar, q, [x for x in X for _ in range(B)], table, B)
        return out["accept_len"] > np.tile(np.arange(B), nx)

    theta = count_below(acc_pred, nx * B).reshape(nx, B).astype(np.float64) / GRID

    # residual token after a rejection at i: accept forced off at i (u just below 1)
    def res_pred(m):  # query (x, i, t)
        table = np.zeros((nx * B * vocab, B + 1, 4))
        table[:, :, oracle.DRAW_TARGET] = 0.5
        ii = np.tile(np.repeat(np.arange(B), vocab), nx)
        for i in range(B):
            sel = ii == i
            table[sel, i, oracle.DRAW_ACCEPT] = 1.0 - 1.0 / GRID
            table[sel, i, oracle.DRAW_RESIDUAL] = u_of(m[sel])
        out = _verify(ar, q, [x for x in X for _ in range(B * vocab)], table, B)
        tt = np.tile(np.arange(vocab), nx * B)
        tok = out["tokens"][np.arange(nx * B * vocab), ii]
        return tok <= tt

    C = count_below(res_pred, nx * B * vocab).reshape(nx, B, vocab)
    res = np.diff(np.concatenate([np.zeros((nx, B, 1), np.int64), C], axis=2), axis=2) / GRID

    # bonus token when every position is accepted
    def bonus_pred(m):  # query (x, t)
        table = np.zeros((nx * vocab, B + 1, 4))
        table[:, B, oracle.DRAW_TARGET] = u_of(m)
        out = _verify(ar, q, [x for x in X for _ in range(vocab)], table, B)
        return out["tokens"][:, B] <= np.tile(np.arange(vocab), nx)

    C = count_below(bonus_pred, nx * vocab).reshape(nx, vocab)
    bonus = np.diff(np.concatenate([np.zeros((nx, 1), np.int64), C], axis=1), axis=1) / GRID

    # emitted prefixes -> completed sequences
    full = np.zeros((vocab,) * (B + 1))
    for a, x in enumerate(X):
        px = np.prod([Pq[i, x[i]] for i in range(B)])
        reach = px
        for m_ in range(B + 1):
            if m_ < B:
                for t in range(vocab):
                    pe = reach * (1.0 - theta[a, m_]) * res[a, m_, t]
                    if pe > 0:
                        _complete_into(full, ar, list(x[:m_]) + [t], pe, B)
                reach *= theta[a, m_]
            else:
                for t in range(vocab):
                    pe = reach * bonus[a, t]
                    if pe > 0:
                        _complete_into(full, ar, list(x) + [t], pe, B)
    return full, ar, (Pq, theta, res, bonus, X)


def _complete_into(full, ar, prefix, pe, B):
    """Add pe * P_AR(rest | prefix) to every completion of prefix to B+1 tokens."""
    rest = B + 1 - len(prefix)
    for tail in itertools.product(range(ar.vocab), repeat=rest):
        seq = prefix + list(tail)
        pr = pe
        for t in range(len(prefix), B + 1):
            pr *= ar.w[tuple(seq[:t])][seq[t]]
            if pr == 0.0:
                break
        if pr > 0.0:
            full[tuple(seq)] += pr


def _ar_table(ar, vocab, B):
    ref = np.zeros((vocab,) * (B + 1))
    for seq in itertools.product(range(vocab), repeat=B + 1):
        ref[seq] = ar.seq_prob(list(seq))
    return ref


LINEAR_CASES = [(4, 3, 4, 1.0, 1), (4, 3, 3, 1.0, 2), (5, 2, 5, 0.97, 3), (8, 2, 4, 0.97, 4), (3, 3, 2, 0.97, 5)]


@pytest.mark.parametrize("vocab,B,top_k,top_p,seed", LINEAR_CASES)
def test_linear_exact_distribution_is_the_target_process(vocab, B, top_k, top_p, seed):
    full, ar, (Pq, theta, res, bonus, X) = linear_exact(vocab, B, top_k, top_p, seed)
    ref = _ar_table(ar, vocab, B)
    assert abs(ref.sum() - 1.0) < 1e-12
    assert np.max(np.abs(full - ref)) < 1e-12
    # the enumeration is not degenerate: some drafts are rejected, some accepted
    assert np.any((theta > 0) & (theta < 1)) or (np.any(theta == 0) and np.any(theta == 1))
    # the measured proposal probabilities are the filtered draft rows
    q_logits, qw = dyadic_rows(B, vocab, top_k, top_p, seed + 1000, min_kept=3)
    assert np.array_equal(Pq, qw)


def test_linear_sampled_output_matches_the_enumeration():
    """The oracle's Philox-driven output (chi-square) against the exact
    distribution from the enumeration."""
    vocab, B, top_k, top_p, seed = 4, 2, 4, 1.0, 7
    full, ar, (Pq, theta, res, bonus, X) = linear_exact(vocab, B, top_k, top_p, seed)
    q_logits, _ = dyadic_rows(B, vocab, top_k, top_p, seed + 1000, min_kept=3)
    R = 100_000
    x = np.ascontiguousarray(np.broadcast_to(q_logits, (R, B, vocab)).reshape(R * B, vocab))
    q = oracle.filter_softmax(x, F32, 1.0, top_k, top_p, rows_per_request=B, rng=(seed, 0))
    drafts = q["sample"].reshape(R, B)
    target = np.stack([np.stack([ar.rows[tuple(drafts[r, :i])] for i in range(B + 1)]) for r in range(R)])
    out = oracle.linear_verify(target.reshape(R * (B + 1), vocab), F32, R, B, 1.0, top_k, top_p, drafts,
                               q["ids"], q["probs"], q["count"], rng=(seed, 0))
    rng = np.random.default_rng(seed)
    seqs = np.full((R, B + 1), -1)
    for r in range(R):
        n = out["num_tokens"][r]
        seqs[r, :n] = out["tokens"][r, :n]
        for t in range(n, B + 1):
            w = ar.w[tuple(seqs[r, :t])]
            seqs[r, t] = int(np.searchsorted(np.cumsum(w), rng.random(), side="right"))
    codes = np.ravel_multi_index(seqs.T, (vocab,) * (B + 1))
    counts = np.bincount(codes, minlength=vocab ** (B + 1))
    assert chi2_pvalue(counts, full.ravel()) > 1e-4


# ---------------------------------------------------------------------------
# Tree verification.
# ---------------------------------------------------------------------------
def tree_exact(vocab, B, K, V, top_k, top_p, seed):
    ar = DyadicAR(vocab, B, top_k, top_p, seed)
    q_logits, _ = dyadic_rows(B, vocab, top_k, top_p, seed + 1000, min_kept=3)
    q = oracle.filter_softmax(q_logits, F32, 1.0, top_k, top_p, rows_per_request=B)
    tree = oracle.tree_topk_expand(q["ids"], q["probs"], q["count"], 1, B, K, V)
    tok, par, dep, nn = tree["node_token"][0], tree["node_parent"][0], tree["node_depth"][0], tree["num_nodes"][0]
    path = {0: ()}
    for j in range(1, nn):
        path[j] = path[par[j]] + (int(tok[j]),)
    one_hot = {}
    for t in range(vocab):
        row = np.full(vocab, -np.inf, dtype=np.float32)
        row[t] = 0.0
        one_hot[t] = row

    # node j's draw, reached by making every ancestor's target row one-hot on
    # the path token (the walk at node j reads only row j and u(j))
    def pred(m):  # query (j, t)
        nqq = nn * vocab
        jj = np.repeat(np.arange(nn), vocab)
        tt = np.tile(np.arange(vocab), nn)
        target = np.zeros((nqq, V, vocab), dtype=np.float32)
        for qi in range(nqq):
            j = jj[qi]
            anc = []
            a = j
            while a > 0:
                anc.append(a)
                a = par[a]
            on_path = {par[c]: tok[c] for c in anc}  # ancestor node -> token of the child on the path
            for n_ in range(V):
                if n_ < nn and n_ != j and n_ in on_path:
                    target[qi, n_] = one_hot[int(on_path[n_])]
                elif n_ < nn:
                    target[qi, n_] = ar.rows[path[n_]]
                else:
                    target[qi, n_] = one_hot[0]
        table = np.full((nqq, V, 4), 0.5)
        table[np.arange(nqq), jj, oracle.DRAW_TARGET] = u_of(m)
        with oracle.injected_uniforms(table):
            out = oracle.tree_verify(target.reshape(nqq * V, vocab), F32, nqq, B, V, 1.0, top_k, top_p,
                                     np.broadcast_to(tok, (nqq, V)).copy(), np.broadcast_to(par, (nqq, V)).copy(),
                                     np.full(nqq, nn, dtype=np.int32), rng=(0, 0))
        got = out["tokens"][np.arange(nqq), dep[jj]]
        return got <= tt

    C = count_below(pred, nn * vocab).reshape(nn, vocab)
    draw = np.diff(np.concatenate([np.zeros((nn, 1), np.int64), C], axis=1), axis=1) / GRID
    children = {j: {int(tok[c]): c for c in range(1, nn) if par[c] == j} for j in range(nn)}
    full = np.zeros((vocab,) * (B + 1))

    def walk(j, reach):
        for t in range(vocab):
            pe = reach * draw[j, t]
            if pe == 0.0:
                continue
            if t in children[j]:
                walk(children[j][t], pe)
            else:
                _complete_into(full, ar, list(path[j]) + [t], pe, B)

    walk(0, 1.0)
    return full, ar, tree, draw


TREE_CASES = [(4, 3, 2, 6, 4, 1.0, 11), (4, 2, 3, 5, 3, 1.0, 12), (5, 2, 2, 4, 5, 0.97, 13), (3, 3, 2, 7, 3, 1.0, 14)]


@pytest.mark.parametrize("vocab,B,K,V,top_k,top_p,seed", TREE_CASES)
def test_tree_exact_distribution_is_the_target_process(vocab, B, K, V, top_k, top_p, seed):
    full, ar, tree, draw = tree_exact(vocab, B, K, V, top_k, top_p, seed)
    ref = _ar_table(ar, vocab, B)
    assert np.max(np.abs(full - ref)) < 1e-12
    assert tree["num_nodes"][0] > 2  # a real tree, not a chain of one
