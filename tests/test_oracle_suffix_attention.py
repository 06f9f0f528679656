"""Pins of the tree-suffix attention and LSE-merge oracle.

The merge of two partial attention states by their log-sum-exps must equal
attention over the union of the two key sets, computed here directly with
``scipy.special.softmax`` / ``logsumexp``; a chain tree must give causal
attention (``torch.nn.functional.scaled_dot_product_attention`` in float64);
grouped key/value heads must equal the same heads repeated.  Each pin takes
the oracle module as an argument so that planted mistakes in a copy of it can
be shown to fail a pin.
"""
import importlib.util
import sys

import numpy as np
import pytest
import torch
from scipy import special

import oracle.suffix_attention as SA


def _case(V, H, Hkv, d, L, seed, parent=None):
    rng = np.random.default_rng(seed)
    if parent is None:
        parent = np.array([-1] + [int(rng.integers(0, j)) for j in range(1, V)])
    q = rng.standard_normal((V, H, d))
    k = rng.standard_normal((V, Hkv, d))
    v = rng.standard_normal((V, Hkv, d))
    kp = rng.standard_normal((L, Hkv, d))
    vp = rng.standard_normal((L, Hkv, d))
    return q, k, v, kp, vp, np.asarray(parent)


def _union_reference(q, k, v, kp, vp, mask, scale):
    """Attention of every node over [prefix keys; visible tree keys]."""
    V, H, d = q.shape
    g = H // k.shape[1]
    o = np.zeros((V, H, d))
    lse = np.zeros((V, H))
    for j in range(V):
        for h in range(H):
            keys = np.concatenate([kp[:, h // g], k[mask[j], h // g]])
            vals = np.concatenate([vp[:, h // g], v[mask[j], h // g]])
            s = scale * keys @ q[j, h]
            o[j, h] = special.softmax(s) @ vals
            lse[j, h] = special.logsumexp(s)
    return o, lse


def pin_merge_equals_union(sa):
    for V, H, Hkv, d, L, seed in [(7, 4, 2, 16, 23, 1), (12, 8, 8, 8, 5, 2), (32, 4, 1, 32, 64, 3)]:
        q, k, v, kp, vp, parent = _case(V, H, Hkv, d, L, seed)
        scale = 1 / np.sqrt(d)
        op, lp = sa.prefix_attention(q, kp, vp, scale)
        o, lse = sa.suffix_attention_merge(q, k, v, parent, op, lp, scale)
        ro, rl = _union_reference(q, k, v, kp, vp, _ancestors(parent), scale)
        assert np.max(np.abs(o - ro)) < 1e-12
        assert np.max(np.abs(lse - rl)) < 1e-12


def _ancestors(parent):
    """Brute force: i is visible from j when walking parents from j reaches i."""
    V = len(parent)
    m = np.zeros((V, V), dtype=bool)
    for j in range(V):
        path, x = set(), j
        for _ in range(V):
            path.add(x)
            if parent[x] < 0:
                break
            x = parent[x]
        for i in path:
            m[j, i] = True
    return m


def pin_chain_tree_is_causal_attention(sa):
    V, H, Hkv, d = 9, 4, 2, 16
    q, k, v, _, _, parent = _case(V, H, Hkv, d, 0, 4, parent=[-1] + list(range(V - 1)))
    scale = 0.3
    o_s, l_s = sa.suffix_attention(q, k, v, parent, scale)
    g = H // Hkv
    tq = torch.from_numpy(q).permute(1, 0, 2)  # [H, V, d]
    tk = torch.from_numpy(np.repeat(k, g, axis=1)).permute(1, 0, 2)
    tv = torch.from_numpy(np.repeat(v, g, axis=1)).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=scale)
    assert np.max(np.abs(o_s - ref.permute(1, 0, 2).numpy())) < 1e-12
    # the LSE of a causal row is the logsumexp of its first j+1 scores
    for j in range(V):
        for h in range(H):
            s = scale * k[:j + 1, h // g] @ q[j, h]
            assert abs(l_s[j, h] - special.logsumexp(s)) < 1e-12


def pin_grouped_heads_equal_repeated_heads(sa):
    V, H, Hkv, d = 6, 8, 2, 8
    q, k, v, kp, vp, parent = _case(V, H, Hkv, d, 11, 5)
    scale = 0.25
    op, lp = sa.prefix_attention(q, kp, vp, scale)
    o, lse = sa.suffix_attention_merge(q, k, v, parent, op, lp, scale)
    g = H // Hkv
    rep = [np.repeat(a, g, axis=1) for a in (k, v, kp, vp)]
    op2, lp2 = sa.prefix_attention(q, rep[2], rep[3], scale)
    o2, lse2 = sa.suffix_attention_merge(q, rep[0], rep[1], parent, op2, lp2, scale)
    assert np.max(np.abs(o - o2)) < 1e-13 and np.max(np.abs(lse - lse2)) < 1e-13
    # and a query head is not paired with another group's key/value head
    k_bad = k.copy()
    k_bad[:, 1] += np.random.default_rng(10).standard_normal(k_bad[:, 1].shape)  # not a uniform shift
    o3, _ = sa.suffix_attention(q, k_bad, v, parent, scale)
    o4, _ = sa.suffix_attention(q, k, v, parent, scale)
    assert np.max(np.abs(o3[:, :g] - o4[:, :g])) < 1e-13  # heads of group 0 do not read kv head 1
    assert np.max(np.abs(o3[:, g:] - o4[:, g:])) > 1e-3


def test_merge_equals_attention_over_the_union():
    pin_merge_equals_union(SA)


def test_chain_tree_is_causal_attention():
    pin_chain_tree_is_causal_attention(SA)


def test_grouped_heads_equal_repeated_heads():
    pin_grouped_heads_equal_repeated_heads(SA)


def test_single_node_and_star_tree():
    q, k, v, _, _, _ = _case(1, 2, 1, 4, 0, 6, parent=[-1])
    o, l = SA.suffix_attention(q, k, v, [-1], 0.5)
    assert np.array_equal(o[0, 0], v[0, 0]) and np.array_equal(o[0, 1], v[0, 0])
    assert abs(l[0, 0] - 0.5 * q[0, 0] @ k[0, 0]) < 1e-14
    V = 5
    m = SA.tree_mask([-1] + [0] * (V - 1))  # every node a child of the root
    assert np.array_equal(m, np.eye(V, dtype=bool) | (np.arange(V)[None, :] == 0))


def test_empty_prefix_leaves_the_suffix():
    q, k, v, kp, vp, parent = _case(6, 4, 2, 8, 0, 7)
    op, lp = SA.prefix_attention(q, kp, vp, 0.3)
    assert np.all(np.isneginf(lp))
    o, lse = SA.suffix_attention_merge(q, k, v, parent, op, lp, 0.3)
    o_s, l_s = SA.suffix_attention(q, k, v, parent, 0.3)
    assert np.array_equal(o, o_s) and np.array_equal(lse, l_s)


def test_merge_is_symmetric_and_associative():
    rng = np.random.default_rng(8)
    parts = [(rng.standard_normal((3, 2, 4)), rng.standard_normal((3, 2)) * 3) for _ in range(3)]
    a, b, c = parts
    ab = SA.lse_merge(*a, *b)
    ba = SA.lse_merge(*b, *a)
    assert np.max(np.abs(ab[0] - ba[0])) < 1e-14 and np.max(np.abs(ab[1] - ba[1])) < 1e-14
    left = SA.lse_merge(*SA.lse_merge(*a, *b), *c)
    right = SA.lse_merge(*a, *SA.lse_merge(*b, *c))
    assert np.max(np.abs(left[0] - right[0])) < 1e-13 and np.max(np.abs(left[1] - right[1])) < 1e-13


def test_bad_trees_and_heads_rejected():
    for parent in ([0, 0], [-1, 1], [-1, 0, 3], [], [-1, -1]):
        with pytest.raises(ValueError):
            SA.tree_mask(parent)
    q, k, v, _, _, parent = _case(3, 4, 3, 4, 0, 9)
    with pytest.raises(ValueError):
        SA.suffix_attention(q, k, v, parent, 1.0)


MUTATIONS = {
    "ancestors taken as every lower index": ("            i = parent[i]\n", "            i = i - 1\n",
                                             pin_merge_equals_union),
    "LSE without its max": ("            lse[j, h] = m + np.log(total)\n", "            lse[j, h] = np.log(total)\n",
                            pin_merge_equals_union),
    "merge weights swapped": ("w1[..., None] * o1 + w2[..., None] * o2", "w2[..., None] * o1 + w1[..., None] * o2",
                              pin_merge_equals_union),
    "heads grouped by modulo": ("np.arange(H) // (H // Hkv)", "np.arange(H) % Hkv",
                                pin_grouped_heads_equal_repeated_heads),
    "scale left out of the suffix": ("            s = scale * (k[seen, kvh[h], :] @ q[j, h, :])\n",
                                     "            s = k[seen, kvh[h], :] @ q[j, h, :]\n",
                                     pin_chain_tree_is_causal_attention),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(name, tmp_path):
    old, new, pin = MUTATIONS[name]
    src = open(SA.__file__).read()
    assert src.count(old) == 1, f"mutation anchor for {name!r} not unique"
    path = tmp_path / "suffix_attention_mut.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location("suffix_attention_mut", path)
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod
    try:
        spec.loader.exec_module(mod)
        with pytest.raises(AssertionError):
            pin(mod)
    finally:
        del sys.modules[spec.name]
