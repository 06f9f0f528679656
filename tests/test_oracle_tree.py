"""Pins of the oracle's tree mode: top-K extraction, best-first expansion and
target-only tree verification."""
import itertools

import numpy as np
import pytest

import oracle
from _defs import chi2_pvalue, filtered_dist
from test_oracle_linear import TinyAR


def _marginals(B, vocab, seed, T=1.0, k=50, p=1.0, scale=1.5):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((B, vocab)) * scale).astype(np.float32)
    return x, oracle.filter_softmax(x, "f32", T, k, p, rows_per_request=B)


def _paths(tree, r=0):
    tok, par, nn = tree["node_token"][r], tree["node_parent"][r], tree["num_nodes"][r]
    out = {}
    for j in range(1, nn):
        path, n = [], j
        while n > 0:
            path.append(int(tok[n]))
            n = par[n]
        out[j] = tuple(reversed(path))
    return out


@pytest.mark.parametrize("B,K,V,seed", [(3, 3, 8, 1), (3, 3, 20, 2), (4, 2, 12, 3), (2, 5, 30, 4)])
def test_expansion_is_the_top_scoring_paths(B, K, V, seed):
    vocab = 9
    _, q = _marginals(B, vocab, seed)
    tree = oracle.tree_topk_expand(q["ids"], q["probs"], q["count"], 1, B, K, V)
    # brute force: every path of length 1..B over each depth's K best tokens
    cand = []
    for d in range(B):
        c = q["count"][d]
        ids, pr = q["ids"][d, :c], q["probs"][d, :c]
        o = np.lexsort((ids, -pr))[:K]
        cand.append(list(zip(ids[o].tolist(), pr[o].tolist())))
    scored = []
    for L in range(1, B + 1):
        for combo in itertools.product(*[range(len(cand[d])) for d in range(L)]):
            s = 1.0
            for d, c in enumerate(combo):
                s *= cand[d][c][1]
            scored.append((s, tuple(cand[d][c][0] for d, c in enumerate(combo))))
    scored.sort(key=lambda t: -t[0])
    n_expected = min(V - 1, len(scored))
    expect = {path for _, path in scored[:n_expected]}
    got = set(_paths(tree).values())
    assert tree["num_nodes"][0] == n_expected + 1
    assert got == expect
    # prefix-closed, parent before child, depth = parent depth + 1, scores non-increasing
    for path in got:
        assert len(path) == 1 or path[:-1] in got
    par, dep, sco = tree["node_parent"][0], tree["node_depth"][0], tree["node_score"][0]
    for j in range(1, tree["num_nodes"][0]):
        assert 0 <= par[j] < j and dep[j] == dep[par[j]] + 1
        assert sco[j] <= sco[j - 1]


def test_k_one_gives_the_argmax_chain():
    B, vocab = 6, 30
    x, q = _marginals(B, vocab, 5)
    tree = oracle.tree_topk_expand(q["ids"], q["probs"], q["count"], 1, B, 1, B + 1)
    assert tree["num_nodes"][0] == B + 1
    assert list(tree["node_parent"][0]) == [-1] + list(range(B))
    assert list(tree["node_token"][0, 1:]) == list(np.argmax(x, axis=1))


def test_ties_break_by_depth_then_parent_then_rank():
    # uniform marginals: every candidate has probability 1/4, so scores tie
    # within a depth and fall with depth
    B, K, V, vocab = 3, 3, 12, 4
    x = np.zeros((B, vocab), dtype=np.float32)
    q = oracle.filter_softmax(x, "f32", 1.0, 50, 1.0, rows_per_request=B)
    tree = oracle.tree_topk_expand(q["ids"], q["probs"], q["count"], 1, B, K, V)
    assert list(tree["node_depth"][0]) == [0, 1, 1, 1, 2, 2, 2, 2, 2, 2, 2, 2]
    assert list(tree["node_parent"][0]) == [-1, 0, 0, 0, 1, 1, 1, 2, 2, 2, 3, 3]
    assert list(tree["node_token"][0]) == [-1, 0, 1, 2, 0, 1, 2, 0, 1, 2, 0, 1]
    # a one-hot second marginal gives each depth-2 child its parent's score,
    # tying it with the remaining depth-1 nodes: the shallower node goes first
    x = np.zeros((2, vocab), dtype=np.float32)
    x[1, 1:] = -np.inf
    q = oracle.filter_softmax(x, "f32", 1.0, 50, 1.0, rows_per_request=2)
    tree = oracle.tree_topk_expand(q["ids"], q["probs"], q["count"], 1, 2, 4, 9)
    assert list(tree["node_depth"][0]) == [0, 1, 1, 1, 1, 2, 2, 2, 2]
    assert list(tree["node_parent"][0]) == [-1, 0, 0, 0, 0, 1, 2, 3, 4]
    assert list(tree["node_token"][0]) == [-1, 0, 1, 2, 3, 0, 0, 0, 0]


def test_tree_shape_constraints_are_rejected():
    _, q = _marginals(4, 10, 6)
    for B, K, V in [(4, 2, 3), (4, 2, 129), (4, 64, 64)]:
        with pytest.raises(oracle.OracleError):
            oracle.tree_topk_expand(q["ids"], q["probs"], q["count"], 1, B, K, V)


def _tree_targets(ar, tree, R):
    V = tree["node_token"].shape[1]
    paths = _paths(tree)
    rows = np.empty((V, ar.vocab), dtype=np.float32)
    for j in range(V):
        pre = () if j == 0 else paths.get(j, ())
        rows[j] = ar.rows[pre]
    return np.ascontiguousarray(np.broadcast_to(rows, (R, V, ar.vocab)).reshape(R * V, ar.vocab))


@pytest.mark.parametrize("vocab,B,K,V,T,k,p,seed", [(4, 2, 2, 5, 1.0, 4, 1.0, 31), (5, 3, 2, 6, 0.9, 4, 0.95, 32)])
def test_tree_output_is_the_target_process(vocab, B, K, V, T, k, p, seed):
    ar = TinyAR(vocab, B, seed)
    _, q = _marginals(B, vocab, seed + 1, T, k, p)
    tree = oracle.tree_topk_expand(q["ids"], q["probs"], q["count"], 1, B, K, V)
    R = 100_000
    tgt = _tree_targets(ar, tree, R)
    tiled = {key: np.ascontiguousarray(np.broadcast_to(tree[key][0], (R, V))) for key in ("node_token", "node_parent")}
    nn = np.full(R, tree["num_nodes"][0], dtype=np.int32)
    out = oracle.tree_verify(tgt, "f32", R, B, V, T, k, p, tiled["node_token"], tiled["node_parent"], nn,
                             rng=(seed, 0))
    acc, ntok, toks = out["accept_len"], out["num_tokens"], out["tokens"]
    assert np.all(ntok == acc + 1) and np.all((acc >= 0) & (acc <= B))
    # complete every emitted prefix to B+1 tokens with the target process
    seqs = np.full((R, B + 1), -1, dtype=np.int64)
    for r in range(R):
        seqs[r, :ntok[r]] = toks[r, :ntok[r]]
    rng = np.random.default_rng(seed + 7)
    for t in range(B + 1):
        need = np.nonzero(seqs[:, t] < 0)[0]
        u = rng.random(need.size)
        for n, r in enumerate(need):
            d = ar.dist(seqs[r, :t], T, k, p)
            seqs[r, t] = min(int(np.searchsorted(np.cumsum(d), u[n] * d.sum(), side="right")), vocab - 1)
    codes = (seqs * (vocab ** np.arange(B + 1))).sum(axis=1)
    counts = np.bincount(codes, minlength=vocab ** (B + 1))
    probs = np.zeros(vocab ** (B + 1))
    for seq in itertools.product(range(vocab), repeat=B + 1):
        probs[int(np.dot(seq, vocab ** np.arange(B + 1)))] = ar.seq_prob(list(seq), T, k, p)
    assert chi2_pvalue(counts, probs) > 1e-4
    # closed form: E[accept_len] = sum over non-root nodes of the target
    # probability of the node's path
    paths = _paths(tree)
    expect = sum(ar.seq_prob(list(path), T, k, p) for path in paths.values())
    a = acc.astype(np.float64)
    assert abs(a.mean() - expect) < 4 * a.std() / np.sqrt(R)
    # path_nodes walk the tree: each next node is a child of the previous
    for r in range(50):
        pn = out["path_nodes"][r]
        assert pn[0] == 0
        for t in range(1, ntok[r]):
            assert tree["node_parent"][0, pn[t]] == pn[t - 1]
            assert tree["node_token"][0, pn[t]] == toks[r, t - 1]


def test_one_hot_targets_walk_greedily():
    vocab, B, K, V = 12, 4, 3, 10
    ar = TinyAR(vocab, B, 41)
    _, q = _marginals(B, vocab, 42)
    tree = oracle.tree_topk_expand(q["ids"], q["probs"], q["count"], 1, B, K, V)
    tgt = _tree_targets(ar, tree, 1)
    out = oracle.tree_verify(tgt, "f32", 1, B, V, 1.0, 1, 1.0, tree["node_token"], tree["node_parent"],
                             tree["num_nodes"], rng=(0, 0))
    # greedy: follow argmax of each node's row while it matches a child
    j, emitted = 0, []
    paths = _paths(tree)
    children = {}
    for c in range(1, tree["num_nodes"][0]):
        children.setdefault(int(tree["node_parent"][0, c]), {})[int(tree["node_token"][0, c])] = c
    while True:
        y = int(np.argmax(tgt[j]))
        emitted.append(y)
        if y in children.get(j, {}):
            j = children[j][y]
        else:
            break
    assert list(out["tokens"][0, :out["num_tokens"][0]]) == emitted
    assert out["accept_len"][0] == len(emitted) - 1
    assert paths is not None
